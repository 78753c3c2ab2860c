"""FP8 scale variants on the GPU against the oracle ("DeepEP 测试目标 API 系统性参考"
§4.2 per_token_cast_to_fp8: one scale per row; §3.3 low_latency_dispatch():
round_scale (power-of-two scales) and use_ue8m0 (exponent-byte scales); §2.1
dispatch(): use_tma_aligned_col_major_sf).

Every valid combination of the EP_SF_* bits (12) through the standalone cast,
ep_dispatch and ep_layout_dispatch: e4m3 rows and scales bit-exact, the scales
checked both through the logical [rows, groups] view and in the raw buffer
(column-major: entry (row, g) at g * ld + row).  Shapes span ragged row counts
(not multiples of the 4- or 16-entry column padding) and nine 128-column
blocks; four formats also run at the full fp8_dispatch size."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import workload
from gpu_util import fp8_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

SF_PER_ROW, SF_POW2, SF_UE8M0, SF_COL_MAJOR = 0x1, 0x2, 0x4, 0x8
FORMATS = [r | p | u | c for r, (p, u), c in itertools.product(
    (0, SF_PER_ROW), ((0, 0), (SF_POW2, 0), (SF_POW2, SF_UE8M0)), (0, SF_COL_MAJOR))]


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def _expected_scales(fmt, s):
    """Logical [rows, groups] expected scales in the stored element type."""
    return oracle.ue8m0_encode(s) if fmt & SF_UE8M0 else s


def _bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def _raw(t, fmt, rows):
    """The scale array as stored: [rows, G] row-major, or [G, ld] column-major."""
    if fmt & SF_COL_MAJOR:
        G = t.shape[1]
        ld = t.stride(1)
        return torch.as_strided(t, (G, ld), (ld, 1)).cpu().numpy()
    return t.contiguous().cpu().numpy()


def _check_scales(fmt, got, exp_logical, rows_cmp=None):
    """Compare a scale view with the expected logical scales (rows_cmp: a row mask)."""
    g = got.cpu().numpy()
    e = exp_logical
    if rows_cmp is not None:
        g, e = g[rows_cmp], e[rows_cmp]
    assert np.array_equal(_bits(g), _bits(e))


@pytest.mark.parametrize("T,H", [(300, 1152), (1, 128), (37, 7168)])
@pytest.mark.parametrize("fmt", FORMATS)
def test_standalone_cast(ep, fmt, T, H):
    rng = np.random.default_rng(fmt * 1000 + T)
    x = workload.to_bf16_bits((rng.standard_normal((T, H)) * np.exp2(rng.integers(-8, 8, (T, 1))))
                              .astype(np.float32))
    q, s = ep.cast_fp8(to_dev_bf16(x), scale_fmt=fmt)
    rq, rs = oracle.cast_fp8(x, per_row=bool(fmt & SF_PER_ROW), round_scale=bool(fmt & SF_POW2))
    assert np.array_equal(fp8_bits(q), rq)
    exp = _expected_scales(fmt, rs)
    _check_scales(fmt, s, exp)
    raw = _raw(s, fmt, T)
    if fmt & SF_COL_MAJOR:
        cm = oracle.scales_col_major(exp)
        assert raw.shape == cm.shape
        assert np.array_equal(_bits(raw[:, :T]), _bits(cm[:, :T]))
    else:
        assert np.array_equal(_bits(raw), _bits(exp))


T, H, E, K = 320, 1152, 64, 6


def _routing(seed):
    rng = np.random.default_rng(seed)
    scores = rng.standard_normal((T, E)) + np.linspace(0, 3, E)[None, :]
    idx = np.argsort(-scores, axis=1, kind="stable")[:, :K].astype(np.int64)
    idx[rng.random((T, K)) < 0.1] = -1
    w = rng.random((T, K)).astype(np.float32)
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32) * 3)
    return idx, w, x


@pytest.mark.parametrize("zero_pad", [True, False])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("fmt", FORMATS)
def test_dispatch_cast_variants(ep, fmt, fused, zero_pad):
    R, A = 8, 128
    idx, w, x = _routing(fmt + 17)
    ref = oracle.layout(idx, w, E, R, A)
    if fused:
        lay, (q, s) = ep.layout_dispatch(to_dev(idx), to_dev(w), to_dev_bf16(x), E, R, A, cast_to_fp8=True,
                                         do_zero_padding=zero_pad, scale_fmt=fmt)
    else:
        lay = ep.layout(to_dev(idx), to_dev(w), E, R, A)
        q, s = ep.dispatch(lay, to_dev_bf16(x), cast_to_fp8=True, do_zero_padding=zero_pad, scale_fmt=fmt)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    Np = int(ref["off"][-1])
    rq, rs = oracle.cast_fp8(x, per_row=bool(fmt & SF_PER_ROW), round_scale=bool(fmt & SF_POW2))
    exp_q = oracle.dispatch_rows(rq, ref, zero_pad)[:Np]
    exp_s = oracle.dispatch_rows(_expected_scales(fmt, rs), ref, zero_pad)[:Np]
    rows = slice(None) if zero_pad else (ref["recv_src"][:Np] >= 0)
    assert np.array_equal(fp8_bits(q[:Np])[rows], exp_q[rows])
    _check_scales(fmt, s[:Np], exp_s, rows)
    if fmt & SF_COL_MAJOR:
        raw = _raw(s, fmt, lay.capacity)
        per16 = 16 if fmt & SF_UE8M0 else 4
        assert raw.shape[1] % per16 == 0 and lay.capacity <= raw.shape[1] < lay.capacity + per16
        assert np.array_equal(_bits(raw[:, :Np].T)[rows], _bits(exp_s)[rows])


@pytest.mark.parametrize("fmt", [SF_PER_ROW, SF_POW2, SF_COL_MAJOR, SF_POW2 | SF_UE8M0 | SF_COL_MAJOR])
def test_full_size_fp8_dispatch(ep, fmt):
    cfg = workload.config("fp8_dispatch")
    inp = workload.inputs(cfg)
    ref = oracle.layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"], cfg["A"])
    lay = ep.layout(to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), cfg["E"], cfg["R"], cfg["A"])
    q, s = ep.dispatch(lay, to_dev_bf16(inp["x"]), cast_to_fp8=True, do_zero_padding=True, scale_fmt=fmt)
    torch.cuda.synchronize()
    Np = int(ref["off"][-1])
    rq, rs = oracle.cast_fp8(inp["x"], per_row=bool(fmt & SF_PER_ROW), round_scale=bool(fmt & SF_POW2))
    assert np.array_equal(fp8_bits(q[:Np]), oracle.dispatch_rows(rq, ref, True)[:Np])
    _check_scales(fmt, s[:Np], oracle.dispatch_rows(_expected_scales(fmt, rs), ref, True)[:Np])


COL_FORMATS = [f for f in FORMATS if f & SF_COL_MAJOR]


@pytest.mark.parametrize("zero_pad", [True, False])
@pytest.mark.parametrize("fmt", COL_FORMATS)
def test_column_major_staged_and_direct(ep, fmt, zero_pad):
    """Column-major scales leave through the workspace's staging area (a
    handle sized by ep_workspace_bytes) or, when the workspace holds only the
    layout's part, one store per scale from the cast kernel.  Both write the
    same bytes everywhere: the oracle's scales on real rows, zeros on padding
    rows with zero padding, and nothing else (a sentinel fill survives on
    padding rows without zero padding and past the rows in use)."""
    R, A = 8, 128
    idx, w, x = _routing(fmt + 91)
    ref = oracle.layout(idx, w, E, R, A)
    Np = int(ref["off"][-1])
    full = ep.workspace_bytes(T, K, E, A)
    outs = []
    for nbytes in (full, full - T * 512):
        lay = ep.Layout(T, K, E, R, A, torch.device("cuda:0"), workspace_nbytes=nbytes)
        ep.layout(to_dev(idx), to_dev(w), E, R, A, out=lay)
        s = ep.scale_tensor(lay.capacity, H, fmt, lay.device)
        raw = torch.as_strided(s, (s.shape[1], s.stride(1)), (s.stride(1), 1))
        raw.view(torch.uint8).fill_(0x5A)
        q, s = ep.dispatch(lay, to_dev_bf16(x), cast_to_fp8=True, do_zero_padding=zero_pad, scale_fmt=fmt,
                           out_scales=s)
        torch.cuda.synchronize()
        assert ep.get_status(lay) == (ep.EP_OK, 0)
        outs.append((fp8_bits(q[:Np]), raw.cpu().numpy().view(np.uint8).copy()))
    (q0, r0), (q1, r1) = outs
    assert np.array_equal(q0, q1)
    assert np.array_equal(r0, r1)
    rq, rs = oracle.cast_fp8(x, per_row=bool(fmt & SF_PER_ROW), round_scale=bool(fmt & SF_POW2))
    exp_s = _expected_scales(fmt, rs)
    raw = r0.view(np.uint32) if exp_s.dtype == np.float32 else r0
    real = ref["recv_src"][:Np] >= 0
    got = raw[:, :Np].T
    assert np.array_equal(_bits(got[real]), _bits(exp_s[ref["recv_src"][:Np][real]]))
    sentinel = 0x5A5A5A5A if exp_s.dtype == np.float32 else 0x5A
    if zero_pad:
        assert (got[~real] == 0).all()
    else:
        assert (got[~real] == sentinel).all()
    assert (raw[:, Np:] == sentinel).all()


def test_column_major_no_alloc_handle(ep):
    """A no-alloc handle takes the staging area from its fixed array when the
    array has room for it; the scales are the oracle's either way."""
    from combine_ep_layout_11_b200 import _lib
    import ctypes
    lib = _lib.load()
    fmt = SF_COL_MAJOR
    R, A = 8, 128
    idx, w, x = _routing(7)
    ref = oracle.layout(idx, w, E, R, A)
    Np = int(ref["off"][-1])
    lay = ep.Layout(T, K, E, R, A, torch.device("cuda:0"), workspace_nbytes=256)   # replaced by the array
    d_idx, d_w = to_dev(idx), to_dev(w)
    rc = lib.ep_layout_no_alloc(ctypes.c_void_p(d_idx.data_ptr()), ctypes.c_void_p(d_w.data_ptr()), T, K, E, R, A,
                                0, lay.ref(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    q, s = ep.dispatch(lay, to_dev_bf16(x), cast_to_fp8=True, do_zero_padding=True, scale_fmt=fmt)
    torch.cuda.synchronize()
    rq, rs = oracle.cast_fp8(x)
    assert np.array_equal(fp8_bits(q[:Np]), oracle.dispatch_rows(rq, ref, True)[:Np])
    _check_scales(fmt, s[:Np], oracle.dispatch_rows(rs, ref, True)[:Np])


@pytest.mark.parametrize("fmt", [SF_COL_MAJOR, SF_COL_MAJOR | SF_POW2 | SF_UE8M0])
def test_column_major_capacity_overflow(ep, fmt):
    """A receive buffer smaller than the layout: both column-major routes write
    exactly the rows below the capacity (the oracle's scales there) and report
    EP_ERR_CAPACITY."""
    R, A, cap = 8, 128, 1000
    idx, w, x = _routing(fmt + 5)
    ref = oracle.layout(idx, w, E, R, A)
    assert int(ref["off"][-1]) > cap
    full = ep.workspace_bytes(T, K, E, A)
    raws = []
    for nbytes in (full, full - T * 512):
        lay = ep.Layout(T, K, E, R, A, torch.device("cuda:0"), capacity=cap, workspace_nbytes=nbytes)
        ep.layout(to_dev(idx), to_dev(w), E, R, A, out=lay)
        s = ep.scale_tensor(cap, H, fmt, lay.device)
        raw = torch.as_strided(s, (s.shape[1], s.stride(1)), (s.stride(1), 1))
        raw.view(torch.uint8).fill_(0x5A)
        q, s = ep.dispatch(lay, to_dev_bf16(x), cast_to_fp8=True, do_zero_padding=True, scale_fmt=fmt, out_scales=s)
        code, _ = ep.get_status(lay)
        assert code == ep.EP_ERR_CAPACITY
        raws.append(raw.cpu().numpy().view(np.uint8).copy())
    assert np.array_equal(raws[0], raws[1])
    rq, rs = oracle.cast_fp8(x, round_scale=bool(fmt & SF_POW2))
    exp_s = oracle.dispatch_rows(_expected_scales(fmt, rs), ref, True)[:cap]
    got = (raws[0].view(np.uint32) if exp_s.dtype == np.float32 else raws[0])[:, :cap].T
    assert np.array_equal(_bits(got), _bits(exp_s))
