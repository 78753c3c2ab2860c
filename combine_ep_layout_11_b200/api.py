"""Thin torch binding of the C ABI (argument marshalling only).

Names follow "DeepEP 测试目标 API 系统性参考": ``layout`` derives the routing
layout (§2.1, the V2 path that needs only topk_idx), ``dispatch`` and ``combine``
take the layout as their handle (§2.1 / §2.2), ``cast_fp8`` is §4.2's per-token
cast with 128-column scale blocks (or the scale variants of §3.3 and §2.1:
per-row, ``round_scale``, ``use_ue8m0``, ``use_tma_aligned_col_major_sf``).
Every step runs in ``libep_b200.so`` on the tensors' CUDA device, on the
current torch stream; torch only allocates memory.
"""
import ctypes

import torch

from . import _lib

EP_OK = 0
EP_ERR_INVALID_ARG = 1
EP_ERR_CAPACITY = 2
EP_ERR_BAD_EXPERT = 3
EP_ERR_TIMEOUT = 4
EP_ERR_CUDA = 5
EP_ERR_UNSUPPORTED = 6
EP_DTYPE_BF16 = 0
EP_DTYPE_FP8_E4M3 = 1
EP_SF_PER_ROW = 0x1
EP_SF_POW2 = 0x2
EP_SF_UE8M0 = 0x4
EP_SF_COL_MAJOR = 0x8


def scale_format(per_token=False, round_scale=False, use_ue8m0=False, use_tma_aligned_col_major_sf=False):
    """EP_SF_* bits from the pages' option names (UE8M0 implies round_scale)."""
    return ((EP_SF_PER_ROW if per_token else 0) | (EP_SF_POW2 if (round_scale or use_ue8m0) else 0)
            | (EP_SF_UE8M0 if use_ue8m0 else 0) | (EP_SF_COL_MAJOR if use_tma_aligned_col_major_sf else 0))


def scale_tensor(rows, hidden, fmt, device):
    """An uninitialised scale array for ``rows`` FP8 rows in format ``fmt``, as a
    logical [rows, groups] view: fp32 or uint8 (UE8M0) elements, row-major, or
    column-major with the leading dimension padded to 16 bytes (stride (1, ld))."""
    nbytes = int(_lib.load().ep_scale_bytes(rows, hidden, fmt))
    if nbytes < 0:
        raise EpError(EP_ERR_INVALID_ARG, "scale format")
    groups = 1 if fmt & EP_SF_PER_ROW else hidden // 128
    dtype = torch.uint8 if fmt & EP_SF_UE8M0 else torch.float32
    if fmt & EP_SF_COL_MAJOR:
        ld = nbytes // (groups * dtype.itemsize) if groups else 0
        return torch.empty((groups, max(ld, 1)), dtype=dtype, device=device).t()[:rows]
    return torch.empty((rows, groups), dtype=dtype, device=device)


class EpError(RuntimeError):
    def __init__(self, code, what):
        msg = _lib.load().ep_status_string(code).decode()
        super().__init__("%s: %s (status %d)" % (what, msg, code))
        self.code = code


def _check(code, what):
    if code != EP_OK:
        raise EpError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def workspace_bytes(num_tokens, num_topk, num_experts, expert_alignment):
    return int(_lib.load().ep_workspace_bytes(num_tokens, num_topk, num_experts, expert_alignment))


def capacity_rows(num_tokens, num_topk, num_experts, expert_alignment):
    """Receive rows that can never overflow: T*K + E*(A-1)."""
    return int(_lib.load().ep_capacity_rows(num_tokens, num_topk, num_experts, expert_alignment))


class Layout:
    """The dispatch / combine handle: routing layout tensors plus the C struct.

    Tensors (device): ``num_recv_tokens_per_expert`` [E], ``expert_offset`` [E+1],
    ``pair_slot`` [T, K], ``recv_src_token`` / ``recv_weight`` /
    ``recv_local_expert`` [capacity], ``workspace`` (bytes).
    """

    def __init__(self, num_tokens, num_topk, num_experts, num_ranks, expert_alignment, device,
                 capacity=None, num_max_tokens_per_rank=0, workspace_nbytes=None):
        T, K, E, A = num_tokens, num_topk, num_experts, expert_alignment
        if capacity is None:
            capacity = capacity_rows(T, K, E, A)
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.num_tokens, self.num_topk, self.num_experts = T, K, E
        self.num_ranks, self.expert_alignment = num_ranks, A
        self.num_max_tokens_per_rank = num_max_tokens_per_rank
        self.capacity = int(capacity)
        self.device = dev
        self.num_recv_tokens_per_expert = torch.empty(E, **i32)
        self.expert_offset = torch.empty(E + 1, **i32)
        # at least one element so the handle never carries a null pointer
        self._pair_slot_buf = torch.empty(max(T * K, 1), **i32)
        self.pair_slot = self._pair_slot_buf[:T * K].view(T, K)
        n = max(self.capacity, 1)
        self.recv_src_token = torch.empty(n, **i32)
        self.recv_weight = torch.empty(n, dtype=torch.float32, device=dev)
        self.recv_local_expert = torch.empty(n, **i32)
        nbytes = workspace_bytes(T, K, E, A) if workspace_nbytes is None else int(workspace_nbytes)
        if nbytes == 0:
            raise EpError(EP_ERR_INVALID_ARG, "workspace size")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)   # zeroed before first use
        s = _lib.EpLayout()
        s.num_recv_tokens_per_expert = self.num_recv_tokens_per_expert.data_ptr()
        s.expert_offset = self.expert_offset.data_ptr()
        s.pair_slot = self._pair_slot_buf.data_ptr()
        s.recv_src_token = self.recv_src_token.data_ptr()
        s.recv_weight = self.recv_weight.data_ptr()
        s.recv_local_expert = self.recv_local_expert.data_ptr()
        s.workspace = self.workspace.data_ptr()
        s.workspace_bytes = nbytes
        s.capacity = self.capacity
        self.struct = s
        self.cumulative_local_expert_recv_stats = None

    def ref(self):
        return ctypes.byref(self.struct)

    def num_recv_rows(self):
        """Rows in use, expert_offset[E] (reads the device: synchronises)."""
        return int(self.expert_offset[-1].item())

    def rank_offsets(self):
        """Start row of each virtual rank's receive region, [R+1] (device tensor)."""
        El = self.num_experts // self.num_ranks
        return self.expert_offset[::El]


def _set_recv_stats(lay, stats):
    """Point the handle at the caller's running per-expert receive counts (or at none)."""
    if stats is not None:
        assert stats.dtype == torch.int32 and stats.is_contiguous() and stats.numel() == lay.num_experts
        assert stats.device == lay.device
    lay.cumulative_local_expert_recv_stats = stats       # kept alive with the handle
    lay.struct.cumulative_local_expert_recv_stats = _ptr(stats)


def layout(topk_idx, topk_weights, num_experts, num_ranks, expert_alignment=1,
           num_max_tokens_per_rank=0, capacity=None, out=None, cumulative_local_expert_recv_stats=None):
    """Compute the routing layout of ``topk_idx`` [T, K] int64 (-1 = unselected).

    ``out`` may be a ``Layout`` of the same sizes to reuse its memory.
    ``cumulative_local_expert_recv_stats``: int32 [E] on the device or None;
    when given, this call's per-expert receive counts are added to it (§2.1).
    """
    L = _lib.load()
    assert topk_idx.dtype == torch.int64 and topk_idx.dim() == 2 and topk_idx.is_contiguous()
    T, K = topk_idx.shape
    if topk_weights is not None:
        assert topk_weights.dtype == torch.float32 and topk_weights.shape == (T, K)
        assert topk_weights.is_contiguous()
    if out is not None:
        assert (out.num_tokens, out.num_topk, out.num_experts) == (T, K, num_experts), "layout size mismatch"
    lay = out if out is not None else Layout(T, K, num_experts, num_ranks, expert_alignment,
                                             topk_idx.device, capacity, num_max_tokens_per_rank)
    _set_recv_stats(lay, cumulative_local_expert_recv_stats)
    _check(L.ep_layout(_ptr(topk_idx), _ptr(topk_weights), T, K, num_experts, num_ranks,
                       expert_alignment, num_max_tokens_per_rank, lay.ref(), _stream(topk_idx.device)),
           "ep_layout")
    return lay


def ll_layout(topk_idx, topk_weights, num_experts, num_ranks, num_max_dispatch_tokens_per_rank, out=None,
              cumulative_local_expert_recv_stats=None):
    """Low-latency fixed-slab layout (§3.3): expert e owns receive rows
    [e*S, (e+1)*S) with S = num_ranks * num_max_dispatch_tokens_per_rank, its
    pairs first (token-major, k-minor), the rest padding.  Returns a ``Layout``
    (capacity E*S) usable by ``dispatch`` and ``combine``."""
    L = _lib.load()
    assert topk_idx.dtype == torch.int64 and topk_idx.dim() == 2 and topk_idx.is_contiguous()
    T, K = topk_idx.shape
    E, R, M = num_experts, num_ranks, num_max_dispatch_tokens_per_rank
    if topk_weights is not None:
        assert topk_weights.dtype == torch.float32 and topk_weights.shape == (T, K)
        assert topk_weights.is_contiguous()
    if out is None:
        nbytes = int(L.ep_ll_workspace_bytes(T, K, E, R, M))
        if nbytes == 0:
            raise EpError(EP_ERR_INVALID_ARG, "workspace size")
        out = Layout(T, K, E, R, 1, topk_idx.device, capacity=E * R * M, num_max_tokens_per_rank=M,
                     workspace_nbytes=nbytes)
    else:
        assert (out.num_tokens, out.num_topk, out.num_experts) == (T, K, E), "layout size mismatch"
    _set_recv_stats(out, cumulative_local_expert_recv_stats)
    _check(L.ep_ll_layout(_ptr(topk_idx), _ptr(topk_weights), T, K, E, R, M, out.ref(), _stream(topk_idx.device)),
           "ep_ll_layout")
    return out


class RankLayout:
    """The handle of the per-token-per-rank layout (§2.1 without do_expand; §3.1's
    V1 layout quantities) plus its extra outputs.

    Tensors (device): ``num_tokens_per_rank`` [R], ``rank_offset`` [R+1],
    ``token_slot`` [T, R] (receive row of (t, r), -1 if t does not reach r),
    ``is_token_in_rank`` bool [T, R], ``num_tokens_per_expert`` and
    ``num_recv_tokens_per_expert`` (aligned) [E], ``recv_src_token`` [capacity],
    ``recv_topk_idx`` int64 / ``recv_topk_weights`` fp32 [capacity, K].
    ``dispatch`` and ``combine`` (without weights: V1's plain sum) take it as
    their handle.
    """

    def __init__(self, num_tokens, num_topk, num_experts, num_ranks, expert_alignment, device, capacity=None):
        T, K, E, R = num_tokens, num_topk, num_experts, num_ranks
        if capacity is None:
            capacity = T * R
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.num_tokens, self.num_topk, self.num_experts, self.num_ranks = T, K, E, R
        self.expert_alignment = expert_alignment
        self.capacity = int(capacity)
        self.device = dev
        n = max(self.capacity, 1)
        self.num_tokens_per_rank = torch.empty(R, **i32)
        self.rank_offset = torch.empty(R + 1, **i32)
        self._token_slot_buf = torch.empty(max(T * R, 1), **i32)
        self.token_slot = self._token_slot_buf[:T * R].view(T, R)
        self._in_rank_buf = torch.empty(max(T * R, 1), dtype=torch.uint8, device=dev)
        self.is_token_in_rank = self._in_rank_buf[:T * R].view(T, R).view(torch.bool)
        self.num_tokens_per_expert = torch.empty(E, **i32)
        self.num_recv_tokens_per_expert = torch.empty(E, **i32)
        self.recv_src_token = torch.empty(n, **i32)
        self.recv_topk_idx = torch.empty((n, K), dtype=torch.int64, device=dev)
        self.recv_topk_weights = torch.empty((n, K), dtype=torch.float32, device=dev)
        nbytes = int(_lib.load().ep_rank_workspace_bytes(T, R, E))
        if nbytes == 0:
            raise EpError(EP_ERR_INVALID_ARG, "workspace size")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)   # zeroed before first use
        st = _lib.EpLayout()
        st.num_recv_tokens_per_expert = self.num_tokens_per_rank.data_ptr()
        st.expert_offset = self.rank_offset.data_ptr()
        st.pair_slot = self._token_slot_buf.data_ptr()
        st.recv_src_token = self.recv_src_token.data_ptr()
        st.workspace = self.workspace.data_ptr()
        st.workspace_bytes = nbytes
        st.capacity = self.capacity
        self.struct = st

    def ref(self):
        return ctypes.byref(self.struct)

    def num_recv_rows(self):
        """Rows in use, rank_offset[R] (reads the device: synchronises)."""
        return int(self.rank_offset[-1].item())


def rank_layout(topk_idx, topk_weights, num_experts, num_ranks, expert_alignment=1, capacity=None, out=None):
    """Per-token-per-rank layout of ``topk_idx`` [T, K] int64 (§2.1 default
    receive form; §3.1 num_tokens_per_rank / is_token_in_rank /
    num_tokens_per_expert).  ``out`` may be a ``RankLayout`` of the same sizes."""
    L = _lib.load()
    assert topk_idx.dtype == torch.int64 and topk_idx.dim() == 2 and topk_idx.is_contiguous()
    T, K = topk_idx.shape
    if topk_weights is not None:
        assert topk_weights.dtype == torch.float32 and topk_weights.shape == (T, K)
        assert topk_weights.is_contiguous()
    if out is not None:
        assert (out.num_tokens, out.num_topk, out.num_experts, out.num_ranks) == (T, K, num_experts, num_ranks)
    lay = out if out is not None else RankLayout(T, K, num_experts, num_ranks, expert_alignment,
                                                 topk_idx.device, capacity)
    lay.expert_alignment = expert_alignment
    _check(L.ep_rank_layout(_ptr(topk_idx), _ptr(topk_weights), T, K, num_experts, num_ranks, expert_alignment,
                            _ptr(lay._in_rank_buf), _ptr(lay.num_tokens_per_expert),
                            _ptr(lay.num_recv_tokens_per_expert), _ptr(lay.recv_topk_idx),
                            _ptr(lay.recv_topk_weights), lay.ref(), _stream(topk_idx.device)), "ep_rank_layout")
    return lay


def dispatch(lay, x, x_scales=None, cast_to_fp8=False, do_zero_padding=False, out=None, out_scales=None,
             scale_fmt=0):
    """Scatter token rows into the receive buffer (§2.1 dispatch()).

    ``x``: bf16 [T, H], or float8_e4m3fn [T, H] with ``x_scales`` fp32 [T, H/128].
    Returns ``recv_x`` [capacity, H] (bf16, or e4m3 when the input is FP8 or
    ``cast_to_fp8``) and, for FP8 output, ``recv_scales`` [capacity, groups]
    (fp32 per 128-column block unless ``scale_fmt``, EP_SF_* bits from
    ``scale_format()``, asks for another form of the cast's scales).
    """
    L = _lib.load()
    assert x.dim() == 2 and x.is_contiguous() and x.shape[0] == lay.num_tokens
    H = x.shape[1]
    fp8_in = x.dtype == torch.float8_e4m3fn
    assert fp8_in or x.dtype == torch.bfloat16
    fp8_out = fp8_in or cast_to_fp8
    cap = max(lay.capacity, 1)
    if out is None:
        out = torch.empty((cap, H), dtype=torch.float8_e4m3fn if fp8_out else torch.bfloat16, device=x.device)
    if fp8_out and out_scales is None:
        out_scales = scale_tensor(cap, H, scale_fmt, x.device)
    _check(L.ep_dispatch(lay.ref(), _ptr(x), EP_DTYPE_FP8_E4M3 if fp8_in else EP_DTYPE_BF16,
                         _ptr(x_scales if fp8_in else None), H, int(bool(cast_to_fp8)), int(scale_fmt),
                         int(bool(do_zero_padding)), _ptr(out), _ptr(out_scales if fp8_out else None),
                         _stream(x.device)), "ep_dispatch")
    return (out, out_scales) if fp8_out else out


def layout_dispatch(topk_idx, topk_weights, x, num_experts, num_ranks, expert_alignment=1,
                    num_max_tokens_per_rank=0, x_scales=None, cast_to_fp8=False, do_zero_padding=False,
                    capacity=None, out_layout=None, out=None, out_scales=None,
                    cumulative_local_expert_recv_stats=None, scale_fmt=0):
    """Layout and dispatch in one call (§2.1: V2's dispatch() derives the layout
    from topk_idx).  Same results as ``layout`` then ``dispatch``; returns
    ``(layout, recv_x)`` or ``(layout, (recv_x, recv_scales))`` for FP8 output."""
    L = _lib.load()
    assert topk_idx.dtype == torch.int64 and topk_idx.dim() == 2 and topk_idx.is_contiguous()
    T, K = topk_idx.shape
    if topk_weights is not None:
        assert topk_weights.dtype == torch.float32 and topk_weights.shape == (T, K)
        assert topk_weights.is_contiguous()
    assert x.dim() == 2 and x.is_contiguous() and x.shape[0] == T
    if out_layout is not None:
        assert (out_layout.num_tokens, out_layout.num_topk, out_layout.num_experts) == (T, K, num_experts)
    lay = out_layout if out_layout is not None else Layout(T, K, num_experts, num_ranks, expert_alignment,
                                                           topk_idx.device, capacity, num_max_tokens_per_rank)
    _set_recv_stats(lay, cumulative_local_expert_recv_stats)
    H = x.shape[1]
    fp8_in = x.dtype == torch.float8_e4m3fn
    assert fp8_in or x.dtype == torch.bfloat16
    fp8_out = fp8_in or cast_to_fp8
    cap = max(lay.capacity, 1)
    if out is None:
        out = torch.empty((cap, H), dtype=torch.float8_e4m3fn if fp8_out else torch.bfloat16, device=x.device)
    if fp8_out and out_scales is None:
        out_scales = scale_tensor(cap, H, scale_fmt, x.device)
    _check(L.ep_layout_dispatch(_ptr(topk_idx), _ptr(topk_weights), T, K, num_experts, num_ranks,
                                expert_alignment, num_max_tokens_per_rank, lay.ref(), _ptr(x),
                                EP_DTYPE_FP8_E4M3 if fp8_in else EP_DTYPE_BF16, _ptr(x_scales if fp8_in else None),
                                H, int(bool(cast_to_fp8)), int(scale_fmt), int(bool(do_zero_padding)), _ptr(out),
                                _ptr(out_scales if fp8_out else None), _stream(x.device)), "ep_layout_dispatch")
    return lay, ((out, out_scales) if fp8_out else out)


def combine(lay, y, topk_weights=None, bias=None, out=None):
    """Weighted (or, with no weights, plain) ordered reduction back to [T, H] bf16 (§2.2).

    ``bias``: None, a bf16 [T, H] tensor, or a pair of them (§2.2 combine():
    0, 1 or 2 output biases); the fp32 sum starts from bias0 (+ bias1).
    """
    L = _lib.load()
    assert y.dtype == torch.bfloat16 and y.dim() == 2 and y.is_contiguous()
    H = y.shape[1]
    if topk_weights is not None:
        assert topk_weights.dtype == torch.float32 and topk_weights.is_contiguous()
    if bias is None:
        biases = (None, None)
    elif isinstance(bias, torch.Tensor):
        biases = (bias, None)
    else:
        assert len(bias) == 2, "bias is a tensor or a pair of tensors"
        biases = tuple(bias)
    for b in biases:
        if b is not None:
            assert b.dtype == torch.bfloat16 and b.is_contiguous() and b.shape == (lay.num_tokens, H)
    if out is None:
        out = torch.empty((lay.num_tokens, H), dtype=torch.bfloat16, device=y.device)
    _check(L.ep_combine(lay.ref(), _ptr(y), H, _ptr(topk_weights), _ptr(biases[0]), _ptr(biases[1]),
                        _ptr(out), _stream(y.device)), "ep_combine")
    return out


def cast_fp8(x, out=None, out_scales=None, scale_fmt=0):
    """bf16 [T, H] -> (float8_e4m3fn [T, H], scales [T, groups]) (§4.2); fp32
    scales per 128-column block unless ``scale_fmt`` (EP_SF_* bits) says otherwise."""
    L = _lib.load()
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    T, H = x.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.float8_e4m3fn, device=x.device)
    if out_scales is None:
        out_scales = scale_tensor(T, H, scale_fmt, x.device)
    _check(L.ep_cast_fp8(_ptr(x), T, H, int(scale_fmt), _ptr(out), _ptr(out_scales), _stream(x.device)),
           "ep_cast_fp8")
    return out, out_scales


def get_status(lay):
    """(status code, EP_DEV_* flags) of the handle's device status word; synchronises the stream."""
    L = _lib.load()
    flags = ctypes.c_uint32(0)
    code = L.ep_get_status(lay.ref(), _stream(lay.device), ctypes.byref(flags))
    return code, flags.value


def selftest_bounded_wait(lay, timeout_ns):
    _check(_lib.load().ep_selftest_bounded_wait(lay.ref(), int(timeout_ns), _stream(lay.device)),
           "ep_selftest_bounded_wait")
