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


# The library sees only pointers, so the binding checks what a pointer cannot
# carry before it crosses: the tensor's device, dtype, shape and density, and
# that an output is large enough for every row the kernels may write.  A
# failed check raises the same EpError(EP_ERR_INVALID_ARG) a rejected call
# does, and nothing is enqueued.
def _require(ok, what):
    if not ok:
        raise EpError(EP_ERR_INVALID_ARG, what)


def _handle_device(device):
    """torch.device with the index filled in ('cuda' -> the current CUDA device)."""
    dev = torch.device(device)
    if dev.type == "cuda" and dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    return dev


def _check_tensor(t, what, device, dtype=None, shape=None, dense=True):
    _require(isinstance(t, torch.Tensor), "%s must be a tensor" % what)
    _require(t.device.type == "cuda" and t.device == device,
             "%s must be a CUDA tensor on %s, not on %s" % (what, device, t.device))
    if dtype is not None:
        _require(t.dtype == dtype, "%s must be %s, not %s" % (what, dtype, t.dtype))
    if shape is not None:
        _require(tuple(t.shape) == tuple(shape), "%s must have shape %s, not %s" % (what, tuple(shape), tuple(t.shape)))
    if dense:
        _require(t.is_contiguous(), "%s must be contiguous" % what)


def _bytes_from_start(t):
    """Bytes of t's storage from its first element on: all a kernel given t.data_ptr() may reach."""
    return t.untyped_storage().nbytes() - t.storage_offset() * t.element_size()


def _check_routing(topk_idx, topk_weights):
    """topk_idx int64 [T, K] on a CUDA device; topk_weights None or fp32 [T, K] beside it."""
    _require(isinstance(topk_idx, torch.Tensor) and topk_idx.dim() == 2, "topk_idx must be a [T, K] tensor")
    _check_tensor(topk_idx, "topk_idx", topk_idx.device, torch.int64)
    if topk_weights is not None:
        _check_tensor(topk_weights, "topk_weights", topk_idx.device, torch.float32, topk_idx.shape)
    return topk_idx.shape


def _check_scales_out(out_scales, rows, hidden, fmt, device):
    """A caller's scale array: on the device, of the format's element type, and
    holding ep_scale_bytes(rows, hidden, fmt) bytes from its first element."""
    nbytes = int(_lib.load().ep_scale_bytes(rows, hidden, fmt))
    _require(nbytes >= 0, "scale format")
    dtype = torch.uint8 if fmt & EP_SF_UE8M0 else torch.float32
    _check_tensor(out_scales, "out_scales", device, dtype, dense=False)
    _require(_bytes_from_start(out_scales) >= nbytes,
             "out_scales holds %d bytes, the format needs %d" % (_bytes_from_start(out_scales), nbytes))


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
        dev = _handle_device(device)
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
        _check_tensor(stats, "cumulative_local_expert_recv_stats", lay.device, torch.int32, (lay.num_experts,))
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
    T, K = _check_routing(topk_idx, topk_weights)
    if out is not None:
        _require((out.num_tokens, out.num_topk, out.num_experts) == (T, K, num_experts), "layout size mismatch")
        _require(out.device == topk_idx.device, "the layout handle is on another device")
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
    T, K = _check_routing(topk_idx, topk_weights)
    E, R, M = num_experts, num_ranks, num_max_dispatch_tokens_per_rank
    if out is None:
        nbytes = int(L.ep_ll_workspace_bytes(T, K, E, R, M))
        if nbytes == 0:
            raise EpError(EP_ERR_INVALID_ARG, "workspace size")
        out = Layout(T, K, E, R, 1, topk_idx.device, capacity=E * R * M, num_max_tokens_per_rank=M,
                     workspace_nbytes=nbytes)
    else:
        _require((out.num_tokens, out.num_topk, out.num_experts) == (T, K, E), "layout size mismatch")
        _require(out.device == topk_idx.device, "the layout handle is on another device")
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
        dev = _handle_device(device)
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
    T, K = _check_routing(topk_idx, topk_weights)
    if out is not None:
        _require((out.num_tokens, out.num_topk, out.num_experts, out.num_ranks) == (T, K, num_experts, num_ranks),
                 "layout size mismatch")
        _require(out.device == topk_idx.device, "the layout handle is on another device")
    lay = out if out is not None else RankLayout(T, K, num_experts, num_ranks, expert_alignment,
                                                 topk_idx.device, capacity)
    lay.expert_alignment = expert_alignment
    _check(L.ep_rank_layout(_ptr(topk_idx), _ptr(topk_weights), T, K, num_experts, num_ranks, expert_alignment,
                            _ptr(lay._in_rank_buf), _ptr(lay.num_tokens_per_expert),
                            _ptr(lay.num_recv_tokens_per_expert), _ptr(lay.recv_topk_idx),
                            _ptr(lay.recv_topk_weights), lay.ref(), _stream(topk_idx.device)), "ep_rank_layout")
    return lay


def _dispatch_buffers(lay, x, x_scales, cast_to_fp8, out, out_scales, scale_fmt):
    """Check dispatch's tensors against the handle and allocate the outputs
    not given; returns (H, fp8_in, fp8_out, recv_x, recv_scales)."""
    dev, T = lay.device, lay.num_tokens
    _require(isinstance(x, torch.Tensor) and x.dim() == 2 and x.shape[0] == T, "x must be a [T, H] tensor")
    _check_tensor(x, "x", dev)
    H = x.shape[1]
    fp8_in = x.dtype == torch.float8_e4m3fn
    _require(fp8_in or x.dtype == torch.bfloat16, "x must be bfloat16 or float8_e4m3fn, not %s" % x.dtype)
    if fp8_in:
        _require(x_scales is not None, "FP8 input needs x_scales")
        _check_tensor(x_scales, "x_scales", dev, torch.float32, (T, H // 128))
    fp8_out = fp8_in or bool(cast_to_fp8)
    out_dtype = torch.float8_e4m3fn if fp8_out else torch.bfloat16
    cap = max(lay.capacity, 1)
    if out is None:
        out = torch.empty((cap, H), dtype=out_dtype, device=dev)
    else:
        _check_tensor(out, "out", dev, out_dtype)
        _require(out.dim() == 2 and out.shape[1] == H and out.shape[0] >= lay.capacity,
                 "out must be [rows >= capacity %d, H %d], not %s" % (lay.capacity, H, tuple(out.shape)))
    if fp8_out:
        if out_scales is None:
            out_scales = scale_tensor(cap, H, scale_fmt, dev)
        else:
            _check_scales_out(out_scales, lay.capacity, H, scale_fmt, dev)
    return H, fp8_in, fp8_out, out, out_scales


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
    H, fp8_in, fp8_out, out, out_scales = _dispatch_buffers(lay, x, x_scales, cast_to_fp8, out, out_scales, scale_fmt)
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
    T, K = _check_routing(topk_idx, topk_weights)
    if out_layout is not None:
        _require((out_layout.num_tokens, out_layout.num_topk, out_layout.num_experts) == (T, K, num_experts),
                 "layout size mismatch")
        _require(out_layout.device == topk_idx.device, "the layout handle is on another device")
    lay = out_layout if out_layout is not None else Layout(T, K, num_experts, num_ranks, expert_alignment,
                                                           topk_idx.device, capacity, num_max_tokens_per_rank)
    _set_recv_stats(lay, cumulative_local_expert_recv_stats)
    H, fp8_in, fp8_out, out, out_scales = _dispatch_buffers(lay, x, x_scales, cast_to_fp8, out, out_scales, scale_fmt)
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
    dev, T = lay.device, lay.num_tokens
    if bias is None:
        biases = (None, None)
    elif isinstance(bias, torch.Tensor):
        biases = (bias, None)
    else:
        biases = tuple(bias)
        _require(len(biases) == 2, "bias is a tensor or a pair of tensors")
    _require(isinstance(y, torch.Tensor) and y.dim() == 2, "y must be a [rows, H] tensor")
    _check_tensor(y, "y", dev, torch.bfloat16)
    H = y.shape[1]
    if topk_weights is not None:
        _check_tensor(topk_weights, "topk_weights", dev, torch.float32, (T, lay.num_topk))
    for b in biases:
        if b is not None:
            _check_tensor(b, "bias", dev, torch.bfloat16, (T, H))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    else:
        _check_tensor(out, "out", dev, torch.bfloat16, (T, H))
    _check(L.ep_combine(lay.ref(), _ptr(y), H, _ptr(topk_weights), _ptr(biases[0]), _ptr(biases[1]),
                        _ptr(out), _stream(dev)), "ep_combine")
    return out


def cast_fp8(x, out=None, out_scales=None, scale_fmt=0):
    """bf16 [T, H] -> (float8_e4m3fn [T, H], scales [T, groups]) (§4.2); fp32
    scales per 128-column block unless ``scale_fmt`` (EP_SF_* bits) says otherwise."""
    L = _lib.load()
    _require(isinstance(x, torch.Tensor) and x.dim() == 2, "x must be a [T, H] tensor")
    _check_tensor(x, "x", x.device, torch.bfloat16)
    T, H = x.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.float8_e4m3fn, device=x.device)
    else:
        _check_tensor(out, "out", x.device, torch.float8_e4m3fn, (T, H))
    if out_scales is None:
        out_scales = scale_tensor(T, H, scale_fmt, x.device)
    else:
        _check_scales_out(out_scales, T, H, scale_fmt, x.device)
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


# --------------------------------------------------------------------------
# Several source groups (GPUs): receive regions as separate buffers
# --------------------------------------------------------------------------
def source_offsets(counts, num_ranks, expert_alignment, group):
    """Host side of a dispatch from several source groups (§2.1 across ranks).

    ``counts``: host int32 [G, E], row g = source group g's per-expert pair
    counts (what an all-gather of every group's ``num_recv_tokens_per_expert``
    delivers).  Returns ``(row_delta, region_rows, pad_list)`` for ``group``:
    int32 [E], int64 [R] and int64 [P] numpy arrays (see ep_source_offsets)."""
    import numpy as np
    L = _lib.load()
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    _require(counts.ndim == 2, "counts must be [G, E]")
    G, E = counts.shape
    delta = np.zeros(E, np.int32)
    rows = np.zeros(max(num_ranks, 1), np.int64)
    npad = ctypes.c_int64(0)
    args = (ctypes.c_void_p(counts.ctypes.data), G, E, num_ranks, expert_alignment, group,
            ctypes.c_void_p(delta.ctypes.data), ctypes.c_void_p(rows.ctypes.data))
    _check(L.ep_source_offsets(*args, None, 0, ctypes.byref(npad)), "ep_source_offsets")
    pads = np.zeros(max(npad.value, 1), np.int64)
    _check(L.ep_source_offsets(*args, ctypes.c_void_p(pads.ctypes.data), npad.value, ctypes.byref(npad)),
           "ep_source_offsets")
    return delta, rows[:num_ranks], pads[:npad.value]


class RegionTable:
    """The regions of a dispatch / combine across source groups: R bf16
    [capacity, H] tensors of one capacity and width, and the device array of
    their addresses the kernels index.  Build it once and pass it to every
    call (``dispatch_regions`` / ``combine_regions`` also take the list and
    build a table per call, which costs a host-to-device copy)."""

    def __init__(self, regions):
        _require(len(regions) > 0, "no regions")
        device = regions[0].device
        cap, H = regions[0].shape[0], regions[0].shape[-1]
        for r in regions:
            _check_tensor(r, "region", device, torch.bfloat16)
            _require(r.dim() == 2 and tuple(r.shape) == (cap, H),
                     "every region must be bf16 [capacity, H] with one capacity and width")
        self.regions = list(regions)         # kept alive with the table
        self.device = device
        self.capacity, self.hidden = int(cap), int(H)
        self.table = torch.tensor([r.data_ptr() for r in regions], dtype=torch.int64, device=device)

    def __len__(self):
        return len(self.regions)


def _region_table(regions):
    return regions if isinstance(regions, RegionTable) else RegionTable(regions)


def _check_region_call(lay, topk_idx, row_delta, table):
    _require(isinstance(lay, Layout) and lay.expert_alignment == 1, "needs a handle of ep_layout with alignment 1")
    _require(len(table) == lay.num_ranks, "one region per rank (%d)" % lay.num_ranks)
    _require(table.device == lay.device, "the regions are on another device")
    _check_tensor(topk_idx, "topk_idx", lay.device, torch.int64, (lay.num_tokens, lay.num_topk))
    _check_tensor(row_delta, "row_delta", lay.device, torch.int32, (lay.num_experts,))


def dispatch_regions(lay, topk_idx, row_delta, regions, x, pad_list=None):
    """Write this group's bf16 rows into the ranks' regions (a ``RegionTable``,
    or a list of R bf16 [capacity, H] tensors); ``pad_list``: int64 device
    tensor of padding rows to zero-fill, or None.  ``row_delta``: int32 [E]
    device tensor from ``source_offsets``."""
    L = _lib.load()
    rt = _region_table(regions)
    _check_region_call(lay, topk_idx, row_delta, rt)
    _check_tensor(x, "x", lay.device, torch.bfloat16, (lay.num_tokens, rt.hidden))
    table, cap = rt.table, rt.capacity
    n = 0
    if pad_list is not None:
        _check_tensor(pad_list, "pad_list", lay.device, torch.int64)
        n = pad_list.numel()
    _check(L.ep_dispatch_regions(lay.ref(), _ptr(topk_idx), _ptr(row_delta), _ptr(table), cap, _ptr(x),
                                 x.shape[1], _ptr(pad_list) if n else None, n, _stream(lay.device)),
           "ep_dispatch_regions")


def combine_regions(lay, topk_idx, row_delta, regions, topk_weights=None, out=None):
    """Ordered combine of this group's tokens, the rows read from the regions
    (expert outputs: a ``RegionTable`` or a list of R bf16 [capacity, H]
    tensors).  Returns bf16 [T, H]."""
    L = _lib.load()
    rt = _region_table(regions)
    _check_region_call(lay, topk_idx, row_delta, rt)
    table, cap, H = rt.table, rt.capacity, rt.hidden
    if topk_weights is not None:
        _check_tensor(topk_weights, "topk_weights", lay.device, torch.float32, (lay.num_tokens, lay.num_topk))
    if out is None:
        out = torch.empty((lay.num_tokens, H), dtype=torch.bfloat16, device=lay.device)
    _check_tensor(out, "out", lay.device, torch.bfloat16, (lay.num_tokens, H))
    _check(L.ep_combine_regions(lay.ref(), _ptr(topk_idx), _ptr(row_delta), _ptr(table), cap, H,
                                _ptr(topk_weights), _ptr(out), _stream(lay.device)), "ep_combine_regions")
    return out
