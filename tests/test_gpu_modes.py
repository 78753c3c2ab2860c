"""Mode sweep on mid-size inputs, the analogue of test_ep.py's enumerate_ep_modes()
("DeepEP 测试目标 API 系统性参考" §2.1 test coverage: FP8 on/off, alignment
{1, 128}, zero padding, weights, num_bias {0, 1, 2} (one per mode, in turn),
plus -1 entries and rank counts; every layout also adds its counts to a
cumulative_local_expert_recv_stats tensor).  Several
tiles and ragged tails: T = 320 tokens (1920 pairs, 7.5 chunks of 256),
H = 1152 (nine 128-column blocks,
2304-byte bf16 rows), 64 experts, top-6."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import workload
from gpu_util import assert_combine_close, bf16_bits, check_layout, f32_bits, fp8_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

T, H, E, K = 320, 1152, 64, 6


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def _inputs(R, drop, seed):
    rng = np.random.default_rng(seed)
    scores = rng.standard_normal((T, E)) + np.linspace(0, 3, E)[None, :] * (seed % 2)
    idx = np.argsort(-scores, axis=1, kind="stable")[:, :K].astype(np.int64)
    if drop:
        idx[rng.random((T, K)) < drop] = -1
    w = rng.random((T, K)).astype(np.float32)
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32) * 3)
    return idx, w, x


MODES = list(itertools.product([False, True], [1, 128], [False, True], [True, False], [0.0, 0.1], [1, 2, 8, 64]))


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("fp8,A,zero_pad,weighted,drop,R", MODES)
def test_mode(ep, fp8, A, zero_pad, weighted, drop, R, fused):
    mode = (fp8, A, zero_pad, weighted, drop, R)
    seed = hash(mode) % (1 << 20)
    num_bias = MODES.index(mode) % 3
    idx, w, x = _inputs(R, drop, seed)
    wt = w if weighted else None
    ref = oracle.layout(idx, wt, E, R, A)
    xd = to_dev_bf16(x)
    stats0 = np.random.default_rng(seed).integers(0, 1000, E).astype(np.int32)
    stats = to_dev(stats0)
    if fused:
        lay, res = ep.layout_dispatch(to_dev(idx), None if wt is None else to_dev(wt), xd, E, R, A,
                                      cast_to_fp8=fp8, do_zero_padding=zero_pad,
                                      cumulative_local_expert_recv_stats=stats)
        if fp8:
            q, s = res
        else:
            recv = res
    else:
        lay = ep.layout(to_dev(idx), None if wt is None else to_dev(wt), E, R, A,
                        cumulative_local_expert_recv_stats=stats)
        if fp8:
            q, s = ep.dispatch(lay, xd, cast_to_fp8=True, do_zero_padding=zero_pad)
        else:
            recv = ep.dispatch(lay, xd, do_zero_padding=zero_pad)
    Np = int(ref["off"][-1])
    y = workload.expert_outputs(dict(seed=seed, H=H), Np)
    biases = [workload.expert_outputs(dict(seed=seed, H=H), T, seed_offset=1 + i) for i in range(num_bias)]
    bias_arg = None if num_bias == 0 else (to_dev_bf16(biases[0]) if num_bias == 1
                                           else tuple(to_dev_bf16(b) for b in biases))
    out = ep.combine(lay, to_dev_bf16(y), None if wt is None else to_dev(wt), bias=bias_arg)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    check_layout(lay, ref)
    assert np.array_equal(stats.cpu().numpy(), oracle.accumulate_recv_stats(stats0, ref["cnt"]))
    real = ref["recv_src"][:Np] >= 0
    cmp_rows = slice(None) if zero_pad else real
    if fp8:
        rq, rs = oracle.cast_fp8(x)
        eq, es = oracle.dispatch_rows(rq, ref, zero_pad)[:Np], oracle.dispatch_rows(rs, ref, zero_pad)[:Np]
        assert np.array_equal(fp8_bits(q[:Np])[cmp_rows], eq[cmp_rows])
        assert np.array_equal(f32_bits(s[:Np])[cmp_rows], es.view(np.uint32)[cmp_rows])
    else:
        er = oracle.dispatch_rows(x, ref, zero_pad)[:Np]
        assert np.array_equal(bf16_bits(recv[:Np])[cmp_rows], er[cmp_rows])
    exp = oracle.combine(y, ref["pair_slot"], wt, *(biases + [None] * (2 - num_bias)))
    assert assert_combine_close(bf16_bits(out), exp) == 1.0
