"""The low-latency fixed-slab layout on the GPU against the oracle
("DeepEP 测试目标 API 系统性参考" §3.3 low_latency_dispatch():
num_max_dispatch_tokens_per_rank, a receive buffer of [E/R, R * max_tokens, H]
per rank; §3.4 low_latency_combine(): a weighted combine).

Layout outputs bit-exact over every slab row (pairs first, then padding rows
with -1 / 0 / -1), dispatch with and without zero padding and with the FP8
cast, the weighted combine, no tokens, an expert overflowing its slab, and
the full decode workload's layout (1 M slab rows)."""
import numpy as np
import pytest
import torch

import oracle
import workload
from gpu_util import DEV, bf16_bits, check_layout, f32_bits, fp8_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def _check_all_rows(lay, ref):
    """check_layout compares rows [0, off[E]); here off[E] = E * S covers every slab row."""
    Np = check_layout(lay, ref)
    assert Np == lay.capacity
    return Np


@pytest.mark.parametrize("M", [32, 45])
@pytest.mark.parametrize("zero_pad", [True, False])
@pytest.mark.parametrize("fp8", [False, True])
def test_ll_dispatch_combine(ep, M, zero_pad, fp8):
    T, H, E, K, R = 256, 1152, 64, 6, 8
    rng = np.random.default_rng(M * 10 + zero_pad * 2 + fp8)
    scores = rng.standard_normal((T, E)) + np.linspace(0, 3, E)[None, :]
    idx = np.argsort(-scores, axis=1, kind="stable")[:, :K].astype(np.int64)
    idx[rng.random((T, K)) < 0.1] = -1
    w = rng.random((T, K)).astype(np.float32)
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    ref = oracle.ll_layout(idx, w, E, R, M)
    stats0 = np.arange(E, dtype=np.int32)
    stats = to_dev(stats0)
    lay = ep.ll_layout(to_dev(idx), to_dev(w), E, R, M, cumulative_local_expert_recv_stats=stats)
    res = ep.dispatch(lay, to_dev_bf16(x), cast_to_fp8=fp8, do_zero_padding=zero_pad)
    Np = int(ref["off"][-1])
    y = workload.expert_outputs(dict(seed=M, H=H), Np)
    out = ep.combine(lay, to_dev_bf16(y), to_dev(w))
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    _check_all_rows(lay, ref)
    assert np.array_equal(stats.cpu().numpy(), oracle.accumulate_recv_stats(stats0, ref["cnt"]))
    rows = slice(None) if zero_pad else (ref["recv_src"] >= 0)
    if fp8:
        rq, rs = oracle.cast_fp8(x)
        assert np.array_equal(fp8_bits(res[0][:Np])[rows], oracle.dispatch_rows(rq, ref, zero_pad)[rows])
        exp_s = oracle.dispatch_rows(rs, ref, zero_pad).view(np.uint32)
        assert np.array_equal(f32_bits(res[1][:Np])[rows], exp_s[rows])
    else:
        assert np.array_equal(bf16_bits(res[:Np])[rows], oracle.dispatch_rows(x, ref, zero_pad)[rows])
    assert np.array_equal(bf16_bits(out), oracle.combine(y, ref["pair_slot"], w))


def test_ll_no_tokens(ep):
    E, R, M, H = 16, 4, 8, 256
    lay = ep.ll_layout(to_dev(np.zeros((0, 4), np.int64)), None, E, R, M)
    recv = ep.dispatch(lay, torch.zeros((0, H), dtype=torch.bfloat16, device=DEV), do_zero_padding=True)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    S = R * M
    assert lay.expert_offset.cpu().tolist() == [e * S for e in range(E + 1)]
    assert lay.num_recv_tokens_per_expert.cpu().sum() == 0
    assert torch.all(lay.recv_src_token == -1) and torch.all(lay.recv_local_expert == -1)
    assert torch.all(recv.view(torch.int16) == 0)


def test_ll_slab_overflow(ep):
    """Repeated experts within tokens: expert 3 gets 2 * 8 = 16 pairs, its slab holds 8."""
    T, K, E, R, M = 8, 2, 8, 2, 4
    idx = np.tile(np.array([[3, 3]], np.int64), (T, 1))
    lay = ep.ll_layout(to_dev(idx), None, E, R, M)
    code, flags = ep.get_status(lay)
    assert code == ep.EP_ERR_CAPACITY and flags & 2
    ps = lay.pair_slot.cpu().numpy()
    S = R * M
    kept = ps[ps >= 0]
    assert sorted(kept.tolist()) == list(range(3 * S, 4 * S))        # the first S pairs fill the slab
    assert (ps.reshape(-1)[:S] >= 0).all() and (ps.reshape(-1)[S:] == -1).all()


def test_ll_full_decode_layout(ep):
    cfg = workload.config("decode")
    inp = workload.inputs(cfg, with_x=False)
    E, R, M = cfg["E"], cfg["R"], cfg["max_tokens_per_rank"]
    ref = oracle.ll_layout(inp["topk_idx"], inp["topk_weights"], E, R, M)
    lay = ep.ll_layout(to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), E, R, M)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    _check_all_rows(lay, ref)
