"""CPU oracle for DeepEP-style MoE dispatch / combine (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product library (``combine_ep_layout_11_b200``) never imports it and has no CPU
fallback; this package in turn never imports the product library.

The arithmetic lives in ``ep_oracle.c`` (plain, single-threaded C, binary32 where
the method fixes binary32).  This module only marshals numpy arrays.  Every
function cites the page section it follows:

* "DeepEP 测试目标 API 系统性参考" (DeepEP test-target API reference), §2.1
  dispatch(), §2.2 combine(), §3.2 Buffer.combine(), §4.1 refs.py, §4.2 math.py;
* "spark_model/layers/ep_dispatch.rs", build_ep_routing_table;
* "URMA" tag page, the count -> prefix-sum placement -> reorder stages.

Pins (see ``tests/test_oracle_*.py``): brute force against a comparison-sort
formulation, the routing-table page's worked examples, the invariants the pages
fix, the full E4M3 code table and torch's float8 conversion, the fp64-exact
combine within the binary32 error bound, and a hand-derived order example.
No oracle function is unpinned.
"""
import contextlib
import ctypes

import numpy as np

from . import build as _build

OK = 0
ERR_INVALID_ARG = 1
ERR_CAPACITY = 2
ERR_BAD_EXPERT = 3
ERR_INDEX_LEN = 10
ERR_WEIGHT_LEN = 11

_lib = None


def lib():
    """Load (building first if needed) the oracle's shared library."""
    global _lib
    if _lib is None:
        _lib = _load(_build.build())
    return _lib


@contextlib.contextmanager
def use_library(path):
    """Temporarily route every oracle call through another build of the oracle
    (the tests use this to show that the pins reject planted mistakes)."""
    global _lib
    saved = _lib
    _lib = _load(path)
    try:
        yield
    finally:
        _lib = saved


def _load(path):
    """Open one build of the oracle library and declare its C signatures."""
    L = ctypes.CDLL(path)
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    L.orc_layout.restype = i32
    L.orc_layout.argtypes = [vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp]
    L.orc_dispatch_rows.restype = None
    L.orc_dispatch_rows.argtypes = [vp, i64, i64, i64, vp, vp, vp, i64, i32, vp]
    L.orc_cast_fp8.restype = None
    L.orc_cast_fp8.argtypes = [vp, i64, i64, i64, ctypes.c_int, vp, vp]
    L.orc_dequant_fp8.restype = None
    L.orc_dequant_fp8.argtypes = [vp, vp, i64, i64, i64, vp]
    L.orc_rank_layout.restype = ctypes.c_int
    L.orc_rank_layout.argtypes = [vp, vp, i64, i64, i64, i64, i64, i64] + [vp] * 9
    L.orc_ue8m0_encode.restype = ctypes.c_int
    L.orc_ue8m0_encode.argtypes = [vp, i64, vp]
    L.orc_ue8m0_decode.restype = None
    L.orc_ue8m0_decode.argtypes = [vp, i64, vp]
    L.orc_combine.restype = None
    L.orc_combine.argtypes = [vp, i64, vp, vp, i64, i64, vp, vp, vp]
    L.orc_accumulate_recv_stats.restype = None
    L.orc_accumulate_recv_stats.argtypes = [vp, i64, vp]
    L.orc_routing_table.restype = i32
    L.orc_routing_table.argtypes = [vp, i64, vp, i64, i64, i64, i64, i64,
                                    vp, vp, vp, vp, vp, vp, vp, vp]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [f32]
    L.orc_e4m3_decode.restype = f32
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    for name in ("orc_e4m3_encode_array", "orc_e4m3_decode_array", "orc_f32_to_bf16_array"):
        getattr(L, name).restype = None
        getattr(L, name).argtypes = [vp, i64, vp]
    return L


def _p(a, dtype=None):
    if a is None:
        return None
    if dtype is not None:
        assert a.dtype == np.dtype(dtype), (a.dtype, dtype)
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


class OracleError(RuntimeError):
    def __init__(self, code, what):
        super().__init__("%s failed with oracle status %d" % (what, code))
        self.code = code


def capacity_rows(T, K, E, A):
    """Worst-case receive rows: every pair plus (A - 1) padding rows per expert."""
    return T * K + E * (A - 1)


def layout(topk_idx, topk_weights, num_experts, num_ranks, expert_alignment,
           num_max_tokens_per_rank=0, capacity=None, slab=0):
    """Expand layout of the selected (token, k) pairs ([API] §2.1, [URMA] prefix placement).

    Returns a dict with ``cnt`` [E], ``off`` [E+1], ``pair_slot`` [T, K],
    ``recv_src`` / ``recv_w`` / ``recv_lexp`` [capacity].  Rows at and beyond
    ``off[E]`` are left at their initial fill (-1 / 0 / -1) and carry no meaning.
    Raises ``OracleError`` with the oracle's status on invalid input.
    """
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int64)
    T, K = topk_idx.shape
    E = int(num_experts)
    if topk_weights is not None:
        topk_weights = np.ascontiguousarray(topk_weights, dtype=np.float32)
        assert topk_weights.shape == (T, K)
    if capacity is None:
        capacity = capacity_rows(T, K, E, expert_alignment)
    cnt = np.zeros(E, np.int32)
    off = np.zeros(E + 1, np.int32)
    pair_slot = np.full((T, K), -1, np.int32)
    recv_src = np.full(max(capacity, 1), -1, np.int32)
    recv_w = np.zeros(max(capacity, 1), np.float32)
    recv_lexp = np.full(max(capacity, 1), -1, np.int32)
    rc = lib().orc_layout(_p(topk_idx), _p(topk_weights), T, K, E, int(num_ranks),
                          int(expert_alignment), int(num_max_tokens_per_rank), int(capacity), int(slab),
                          _p(cnt), _p(off), _p(pair_slot), _p(recv_src), _p(recv_w), _p(recv_lexp))
    if rc != OK:
        raise OracleError(rc, "layout")
    return dict(cnt=cnt, off=off, pair_slot=pair_slot, recv_src=recv_src[:capacity],
                recv_w=recv_w[:capacity], recv_lexp=recv_lexp[:capacity],
                num_experts=E, num_ranks=int(num_ranks), expert_alignment=int(expert_alignment),
                capacity=int(capacity))


def ll_layout(topk_idx, topk_weights, num_experts, num_ranks, num_max_dispatch_tokens_per_rank):
    """Low-latency fixed-slab layout ([API] §3.3): expert e owns rows
    [e * S, (e + 1) * S) with S = R * num_max_dispatch_tokens_per_rank, its pairs
    first (token-major, k-minor), the rest padding; capacity E * S."""
    R, M = int(num_ranks), int(num_max_dispatch_tokens_per_rank)
    S = R * M
    return layout(topk_idx, topk_weights, num_experts, R, 1, M, capacity=int(num_experts) * S, slab=S)


def rank_layout(topk_idx, topk_weights, num_experts, num_ranks, expert_alignment=1, capacity=None):
    """Per-token-per-rank layout ([API] §2.1 with do_expand off; §3.1's V1
    quantities): one receive row per (token, rank) the token reaches.

    Returns a dict with ``num_tokens_per_rank`` [R], ``rank_off`` [R+1],
    ``is_token_in_rank`` bool [T, R], ``token_slot`` [T, R],
    ``num_tokens_per_expert`` / ``num_recv_tokens_per_expert`` (aligned) [E],
    ``recv_src`` [capacity], ``recv_topk_idx`` int64 / ``recv_topk_weights``
    [capacity, K]; plus ``pair_slot`` / ``cnt`` / ``off`` aliases of
    token_slot / num_tokens_per_rank / rank_off so that ``dispatch_rows`` and
    ``combine`` (with K = R and unit weights) serve this form too.
    """
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int64)
    T, K = topk_idx.shape
    E, R = int(num_experts), int(num_ranks)
    if topk_weights is not None:
        topk_weights = np.ascontiguousarray(topk_weights, dtype=np.float32)
        assert topk_weights.shape == (T, K)
    if capacity is None:
        capacity = T * R
    n_rank = np.zeros(R, np.int32)
    rank_off = np.zeros(R + 1, np.int32)
    in_rank = np.zeros((T, R), np.uint8)
    token_slot = np.full((T, R), -1, np.int32)
    n_exp = np.zeros(E, np.int32)
    n_recv = np.zeros(E, np.int32)
    recv_src = np.full(max(capacity, 1), -1, np.int32)
    recv_idx = np.full((max(capacity, 1), K), -1, np.int64)
    recv_w = np.zeros((max(capacity, 1), K), np.float32)
    rc = lib().orc_rank_layout(_p(topk_idx), _p(topk_weights), T, K, E, R, int(expert_alignment), int(capacity),
                               _p(n_rank), _p(rank_off), _p(in_rank), _p(token_slot), _p(n_exp), _p(n_recv),
                               _p(recv_src), _p(recv_idx), _p(recv_w))
    if rc != OK:
        raise OracleError(rc, "rank layout")
    return dict(num_tokens_per_rank=n_rank, rank_off=rank_off, is_token_in_rank=in_rank.astype(bool),
                token_slot=token_slot, num_tokens_per_expert=n_exp, num_recv_tokens_per_expert=n_recv,
                recv_src=recv_src[:capacity], recv_topk_idx=recv_idx[:capacity], recv_topk_weights=recv_w[:capacity],
                pair_slot=token_slot, cnt=n_rank, off=rank_off, num_experts=R, num_ranks=R,
                capacity=int(capacity))


def dispatch_rows(x_rows, lay, do_zero_padding, fill=0xA5):
    """Row scatter ([API] §2.1): ``recv[pair_slot[t, k]] = x_rows[t]``.

    ``x_rows`` is any [T, row_bytes] array viewed as bytes (bf16 row, fp8 row or a
    row of scales).  Rows that no pair writes keep ``fill`` unless they are
    padding rows and ``do_zero_padding`` is set, in which case they are zero.
    """
    x_rows = np.ascontiguousarray(x_rows)
    T = x_rows.shape[0]
    row_bytes = int(np.prod(x_rows.shape[1:], dtype=np.int64)) * x_rows.dtype.itemsize
    xb = x_rows.reshape(T, -1).view(np.uint8) if T else np.zeros((0, row_bytes), np.uint8)
    cap = lay["capacity"]
    recv = np.full((max(cap, 1), row_bytes), fill, np.uint8)
    K = lay["pair_slot"].shape[1]
    lib().orc_dispatch_rows(_p(xb), row_bytes, T, K, _p(lay["pair_slot"]), _p(lay["cnt"]),
                            _p(lay["off"]), lay["num_experts"], int(bool(do_zero_padding)), _p(recv))
    recv = recv[:cap]
    tail = x_rows.shape[1:]
    return recv.view(x_rows.dtype).reshape((cap,) + tail)


def cast_fp8(x_bf16, per_row=False, round_scale=False):
    """E4M3 cast ([API] §4.2): returns (q uint8 [T, H], scales f32 [T, H/128]).

    ``per_row``: one scale per token row ([T, 1]) as §4.2's per_token_cast_to_fp8
    prints it, instead of one per 128-column block.  ``round_scale``: each
    scale rounded up to a power of two ([API] §3.3 round_scale)."""
    x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, H = x_bf16.shape
    assert H % 128 == 0, "FP8 cast needs H % 128 == 0"
    group = H if per_row else 128
    q = np.zeros((T, H), np.uint8)
    s = np.zeros((T, H // group), np.float32)
    lib().orc_cast_fp8(_p(x_bf16), T, H, group, int(bool(round_scale)), _p(q), _p(s))
    return q, s


def dequant_fp8(q, scales):
    """Dequantisation ([API] §4.2): float(q) * scale in binary32; the group
    width is H / scales.shape[1] (128, or H for per-row scales)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    T, H = q.shape
    group = H // scales.shape[1] if scales.ndim == 2 else H
    out = np.zeros((T, H), np.float32)
    lib().orc_dequant_fp8(_p(q), _p(scales), T, H, group, _p(out))
    return out


def ue8m0_encode(scales):
    """Power-of-two fp32 scales as UE8M0 bytes ([API] §3.3 use_ue8m0): 2^k -> k + 127."""
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    out = np.zeros(scales.shape, np.uint8)
    rc = lib().orc_ue8m0_encode(_p(scales), scales.size, _p(out))
    if rc != 0:
        raise OracleError(rc, "UE8M0 needs power-of-two scales")
    return out


def ue8m0_decode(b):
    """UE8M0 bytes to fp32: b -> 2^(b - 127)."""
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.zeros(b.shape, np.float32)
    lib().orc_ue8m0_decode(_p(b), b.size, _p(out))
    return out


def scales_col_major(scales):
    """TMA-aligned column-major placement of row-major scales [rows, G]
    ([API] §2.1 use_tma_aligned_col_major_sf): entry (r, g) goes to g * ld + r
    with ld = rows rounded up to 16 bytes of elements; returns [G, ld], the
    padding entries zero."""
    scales = np.asarray(scales)
    rows, G = scales.shape
    per16 = 16 // scales.dtype.itemsize
    ld = (rows + per16 - 1) // per16 * per16
    out = np.zeros((G, ld), scales.dtype)
    out[:, :rows] = scales.T
    return out


def combine(y_bf16, pair_slot, topk_weights, bias0=None, bias1=None):
    """Ordered weighted reduction ([API] §2.2, §3.2, §4.1): bf16 [T, H].

    ``y_bf16`` holds the expert outputs, one bf16 row per receive row (uint16
    bits, [rows, H]); ``pair_slot`` [T, K] names the row of each pair; NULL
    (None) weights mean unit weights; ``bias0`` / ``bias1`` (bf16 bits [T, H])
    are the optional output bias, the sum's starting value.
    """
    y_bf16 = np.ascontiguousarray(y_bf16, dtype=np.uint16)
    pair_slot = np.ascontiguousarray(pair_slot, dtype=np.int32)
    T, K = pair_slot.shape
    H = y_bf16.shape[1]
    if pair_slot.size:
        assert pair_slot.max() < y_bf16.shape[0]
    if topk_weights is not None:
        topk_weights = np.ascontiguousarray(topk_weights, dtype=np.float32)
        assert topk_weights.shape == (T, K)
    biases = []
    for b in (bias0, bias1):
        if b is not None:
            b = np.ascontiguousarray(b, dtype=np.uint16)
            assert b.shape == (T, H)
        biases.append(b)
    out = np.zeros((T, H), np.uint16)
    lib().orc_combine(_p(y_bf16), H, _p(pair_slot), _p(topk_weights), T, K, _p(biases[0]), _p(biases[1]),
                      _p(out))
    return out


def accumulate_recv_stats(stats, cnt):
    """cumulative_local_expert_recv_stats ([API] §2.1, §3.3): stats += cnt (int32)."""
    stats = np.array(stats, dtype=np.int32, copy=True)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    lib().orc_accumulate_recv_stats(_p(cnt), cnt.size, _p(stats))
    return stats


def routing_table(gate_indices, gate_weights, num_tokens, top_k, local_start, local_end):
    """Local / remote partition of one rank's pairs ("spark_model/layers/ep_dispatch.rs").

    Returns a dict with the six vectors of the page's routing table.  Length
    mismatches raise ``OracleError`` (status 10 for indices, 11 for weights).
    """
    gi = np.ascontiguousarray(gate_indices, dtype=np.int64).ravel()
    gw = np.ascontiguousarray(gate_weights, dtype=np.float32).ravel()
    n = max(gi.size, 1)
    bufs = [np.zeros(n, np.int32), np.zeros(n, np.int32), np.zeros(n, np.float32),
            np.zeros(n, np.int32), np.zeros(n, np.int32), np.zeros(n, np.float32)]
    nl = ctypes.c_int64(0)
    nr = ctypes.c_int64(0)
    rc = lib().orc_routing_table(_p(gi), gi.size, _p(gw), gw.size, int(num_tokens), int(top_k),
                                 int(local_start), int(local_end),
                                 _p(bufs[0]), _p(bufs[1]), _p(bufs[2]), ctypes.byref(nl),
                                 _p(bufs[3]), _p(bufs[4]), _p(bufs[5]), ctypes.byref(nr))
    if rc != OK:
        raise OracleError(rc, "routing_table")
    a, b = nl.value, nr.value
    return dict(local_token_indices=bufs[0][:a], local_expert_ids=bufs[1][:a],
                local_weights=bufs[2][:a], remote_token_indices=bufs[3][:b],
                remote_expert_ids=bufs[4][:b], remote_weights=bufs[5][:b])


def e4m3_encode(v):
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_decode(c):
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.zeros(c.shape, np.float32)
    lib().orc_e4m3_decode_array(_p(c), c.size, _p(out))
    return out


def f32_to_bf16(v):
    """binary32 -> bf16 bits, round to nearest even (the oracle's output rounding)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, np.uint16)
    lib().orc_f32_to_bf16_array(_p(v), v.size, _p(out))
    return out


def bf16_to_f32(b):
    """bf16 bits -> binary32 (exact widening)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def step_layout(inp, cfg, form="expand"):
    """The layout of one step: ``form`` "expand" (the default), "rank" (the
    per-token-per-rank layout) or "ll" (the fixed-slab layout with
    max_tokens_per_rank, or T / R, tokens per rank)."""
    if form == "rank":
        return rank_layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"], cfg["A"])
    if form == "ll":
        return ll_layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"],
                         cfg.get("max_tokens_per_rank", 0) or cfg["T"] // cfg["R"])
    return layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"], cfg["A"],
                  cfg.get("max_tokens_per_rank", 0))


def step(inp, cfg, form="expand"):
    """One pass of the whole path on host arrays: layout, dispatch (with the
    fused cast in FP8 mode) and combine of the given expert outputs.  Used by the
    benchmark's CPU baseline.  ``form`` as for ``step_layout``; the per-rank
    form combines without weights (V1).  Returns (layout, recv rows, combined out)."""
    per_rank = form == "rank"
    if form != "expand":
        lay = step_layout(inp, cfg, form)
    else:
        lay = layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"], cfg["A"],
                     cfg.get("max_tokens_per_rank", 0))
    if cfg.get("fp8"):
        q, s = cast_fp8(inp["x"])
        recv = (dispatch_rows(q, lay, cfg["zero_pad"]), dispatch_rows(s, lay, cfg["zero_pad"]))
    else:
        recv = dispatch_rows(inp["x"], lay, cfg["zero_pad"])
    w = None if per_rank else inp["topk_weights"]
    out = combine(inp["y"], lay["pair_slot"], w, inp.get("bias0"), inp.get("bias1"))
    return lay, recv, out
