"""Randomised parity: 40 seeded configurations drawn over the whole input
space - T, K, E, R, A, H, the share of -1 entries, weights or none, the three
layout forms (expand, per-rank, fixed slab), bf16 rows or the FP8 cast with a
random scale format, zero padding, 0-2 combine biases - each run through the
C ABI and compared with the oracle bit for bit ("DeepEP 测试目标 API 系统性参考"
§2.1, §2.2, §3.1-§3.3, §4.2)."""
import numpy as np
import pytest
import torch

import oracle
import workload
from gpu_util import bf16_bits, check_layout, f32_bits, fp8_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

SF_PER_ROW, SF_POW2, SF_UE8M0, SF_COL_MAJOR = 0x1, 0x2, 0x4, 0x8


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def draw(seed):
    rng = np.random.default_rng(1000 + seed)
    R = int(rng.choice([1, 2, 3, 4, 8, 16]))
    E = R * int(rng.integers(1, 9))
    T = R * int(rng.integers(0, 40))
    K = int(rng.integers(1, 10))
    form = ["expand", "rank", "ll"][seed % 3]
    fp8 = bool(rng.integers(0, 2))
    H = 128 * int(rng.integers(1, 6)) if fp8 else 8 * int(rng.integers(1, 80))
    A = int(rng.choice([1, 2, 7, 16]))
    fmt = 0
    if fp8:
        fmt = int(rng.choice([0, SF_PER_ROW, SF_POW2, SF_POW2 | SF_UE8M0, SF_COL_MAJOR,
                              SF_PER_ROW | SF_POW2 | SF_UE8M0 | SF_COL_MAJOR]))
    return dict(R=R, E=E, T=T, K=K, H=H, A=A, form=form, fp8=fp8, fmt=fmt,
                drop=float(rng.choice([0.0, 0.2, 0.9])), weighted=bool(rng.integers(0, 2)),
                zero_pad=bool(rng.integers(0, 2)), nbias=int(rng.integers(0, 3)), rng=rng)


@pytest.mark.parametrize("seed", range(40))
def test_random_config(ep, seed):
    c = draw(seed)
    rng, T, K, E, R, A, H = c["rng"], c["T"], c["K"], c["E"], c["R"], c["A"], c["H"]
    idx = rng.integers(0, E, (T, K)).astype(np.int64)
    idx[rng.random((T, K)) < c["drop"]] = -1
    w = rng.random((T, K)).astype(np.float32) if c["weighted"] else None
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32) * 4)
    dw = None if w is None else to_dev(w)
    M = max(T // R, 1) + 2
    if c["form"] == "expand":
        ref = oracle.layout(idx, w, E, R, A)
        lay = ep.layout(to_dev(idx), dw, E, R, A)
    elif c["form"] == "rank":
        ref = oracle.rank_layout(idx, w, E, R, A)
        lay = ep.rank_layout(to_dev(idx), dw, E, R, A)
    else:
        try:
            ref = oracle.ll_layout(idx, w, E, R, M)
        except oracle.OracleError:
            pytest.skip("an expert overflows its slab (repeated experts); covered by the slab tests")
        lay = ep.ll_layout(to_dev(idx), dw, E, R, M)
    res = ep.dispatch(lay, to_dev_bf16(x), cast_to_fp8=c["fp8"], do_zero_padding=c["zero_pad"], scale_fmt=c["fmt"])
    Np = int(ref["off"][-1])
    y = workload.expert_outputs(dict(seed=seed, H=H), max(Np, 1))
    biases = [workload.expert_outputs(dict(seed=seed, H=H), max(T, 1), seed_offset=1 + i)[:T]
              for i in range(c["nbias"])]
    bias = None if not biases else (to_dev_bf16(biases[0]) if len(biases) == 1
                                    else tuple(to_dev_bf16(b) for b in biases))
    cw = None if c["form"] == "rank" else dw
    out = ep.combine(lay, to_dev_bf16(y), cw, bias=bias)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    if c["form"] == "rank":
        assert np.array_equal(lay.token_slot.cpu().numpy(), ref["token_slot"])
        assert np.array_equal(lay.rank_offset.cpu().numpy(), ref["rank_off"])
        assert np.array_equal(lay.recv_topk_idx[:Np].cpu().numpy(), ref["recv_topk_idx"][:Np])
        assert np.array_equal(lay.num_recv_tokens_per_expert.cpu().numpy(), ref["num_recv_tokens_per_expert"])
    else:
        check_layout(lay, ref)
    rows = slice(None) if c["zero_pad"] else (ref["recv_src"][:Np] >= 0)
    if c["fp8"]:
        q, s = res
        rq, rs = oracle.cast_fp8(x, per_row=bool(c["fmt"] & SF_PER_ROW), round_scale=bool(c["fmt"] & SF_POW2))
        es = oracle.ue8m0_encode(rs) if c["fmt"] & SF_UE8M0 else rs
        assert np.array_equal(fp8_bits(q[:Np])[rows], oracle.dispatch_rows(rq, ref, c["zero_pad"])[:Np][rows])
        got_s = s[:Np].cpu().numpy()
        exp_s = oracle.dispatch_rows(es, ref, c["zero_pad"])[:Np]
        if got_s.dtype == np.float32:
            got_s, exp_s = got_s.view(np.uint32), exp_s.view(np.uint32)
        assert np.array_equal(got_s[rows], exp_s[rows])
    else:
        assert np.array_equal(bf16_bits(res[:Np])[rows], oracle.dispatch_rows(x, ref, c["zero_pad"])[:Np][rows])
    exp = oracle.combine(y, ref["pair_slot"], None if c["form"] == "rank" else w,
                         *(biases + [None] * (2 - len(biases))))
    assert np.array_equal(bf16_bits(out), exp)
