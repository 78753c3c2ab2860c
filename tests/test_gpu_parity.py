"""GPU parity on the five workloads at full size, through the C ABI.

Layout (counts, offsets, pair slots, inverse maps), receive buffers (bf16 rows,
e4m3 rows, scales, zeroed padding) must equal the CPU oracle bit for bit;
combine must be within max abs 1e-2 / max rel 8e-3 of the oracle (and is
expected to be bit-exact, checked separately).  Workloads: "DeepEP 测试目标 API
系统性参考" §2.1 / §2.2 shapes (H = 7168, 256 experts, top-8, skewed gates).
"""
import numpy as np
import pytest
import torch

import oracle
import workload
from gpu_util import (DEV, assert_combine_close, bf16_bits, check_layout, f32_bits, fp8_bits, to_dev,
                      to_dev_bf16)

pytestmark = pytest.mark.gpu

NAMES = ["tiny", "prefill_bf16", "fp8_dispatch", "decode", "large_prefill"]


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def _run(ep, name, layout=True):
    cfg = workload.config(name)
    inp = workload.inputs(cfg)
    ref = oracle.layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"], cfg["A"],
                        cfg["max_tokens_per_rank"])
    idx, w = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    x = to_dev_bf16(inp["x"])
    lay = ep.layout(idx, w, cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"]) if layout else None
    return cfg, inp, ref, x, w, lay


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("name", NAMES)
def test_layout_and_dispatch_bit_exact(ep, name, fused):
    """ep_layout + ep_dispatch, and the single-call ep_layout_dispatch."""
    cfg, inp, ref, x, w, lay = _run(ep, name, layout=not fused)
    if fused:
        lay, res = ep.layout_dispatch(to_dev(inp["topk_idx"]), w, x, cfg["E"], cfg["R"], cfg["A"],
                                      cfg["max_tokens_per_rank"], cast_to_fp8=cfg["fp8"],
                                      do_zero_padding=cfg["zero_pad"])
        if cfg["fp8"]:
            q, s = res
        else:
            recv = res
    elif cfg["fp8"]:
        q, s = ep.dispatch(lay, x, cast_to_fp8=True, do_zero_padding=cfg["zero_pad"])
    else:
        recv = ep.dispatch(lay, x, do_zero_padding=cfg["zero_pad"])
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    Np = check_layout(lay, ref)
    if cfg["fp8"]:
        rq, rs = oracle.cast_fp8(inp["x"])
        exp_q = oracle.dispatch_rows(rq, ref, cfg["zero_pad"])
        exp_s = oracle.dispatch_rows(rs, ref, cfg["zero_pad"])
        got_q, got_s = fp8_bits(q[:Np]), f32_bits(s[:Np])
        assert np.array_equal(got_q, exp_q[:Np])
        assert np.array_equal(got_s, exp_s[:Np].view(np.uint32))
        # dequantised values are then equal bit for bit as well
        assert np.array_equal(oracle.dequant_fp8(got_q, got_s.view(np.float32)).view(np.uint32),
                              oracle.dequant_fp8(exp_q[:Np], exp_s[:Np]).view(np.uint32))
    else:
        exp = oracle.dispatch_rows(inp["x"], ref, cfg["zero_pad"])
        got = bf16_bits(recv[:Np])
        if cfg["zero_pad"] or cfg["A"] == 1:
            assert np.array_equal(got, exp[:Np])
        else:
            real = ref["recv_src"][:Np] >= 0
            assert np.array_equal(got[real], exp[:Np][real])


@pytest.mark.parametrize("name", NAMES)
def test_combine_vs_oracle(ep, name):
    cfg, inp, ref, x, w, lay = _run(ep, name)
    Np = int(ref["off"][-1])
    y_host = workload.expert_outputs(cfg, Np)
    out = ep.combine(lay, to_dev_bf16(y_host), w)
    got = bf16_bits(out)
    exp = oracle.combine(y_host, ref["pair_slot"], inp["topk_weights"])
    exact = assert_combine_close(got, exp)
    assert exact == 1.0, "combine is within tolerance but not bit-exact (%.6f equal)" % exact


@pytest.mark.parametrize("num_bias", [1, 2])
@pytest.mark.parametrize("name", ["prefill_bf16", "decode"])
def test_combine_with_bias_vs_oracle(ep, name, num_bias):
    """§2.2 combine() bias: the sum starts at bias0 (+ bias1), bit-exact with the oracle."""
    cfg, inp, ref, x, w, lay = _run(ep, name)
    Np = int(ref["off"][-1])
    y_host = workload.expert_outputs(cfg, Np)
    biases = [workload.expert_outputs(cfg, cfg["T"], seed_offset=1 + i) for i in range(num_bias)]
    dev_b = [to_dev_bf16(b) for b in biases]
    out = ep.combine(lay, to_dev_bf16(y_host), w, bias=dev_b[0] if num_bias == 1 else tuple(dev_b))
    got = bf16_bits(out)
    exp = oracle.combine(y_host, ref["pair_slot"], inp["topk_weights"], *(biases + [None] * (2 - num_bias)))
    exact = assert_combine_close(got, exp)
    assert exact == 1.0, "combine is within tolerance but not bit-exact (%.6f equal)" % exact


@pytest.mark.parametrize("name", ["prefill_bf16", "decode", "large_prefill"])
def test_identity_experts_reproduce_x(ep, name):
    """combine(dispatch(x)) with weights renormalised over the selected entries is x."""
    cfg, inp, ref, x, w, lay = _run(ep, name)
    recv = ep.dispatch(lay, x, do_zero_padding=cfg["zero_pad"])
    idx = inp["topk_idx"]
    wn = np.where(idx >= 0, inp["topk_weights"], 0).astype(np.float32)
    s = wn.sum(axis=1, keepdims=True)
    wn = np.where(s > 0, wn / np.where(s > 0, s, 1), 0).astype(np.float32)
    out = ep.combine(lay, recv, to_dev(wn))
    has = (idx >= 0).any(axis=1)
    got = bf16_bits(out)
    # the sum starts from +0, so a -0 input element comes back as +0
    expect = np.where(inp["x"] == 0x8000, np.uint16(0), inp["x"])
    assert np.array_equal(got[has], expect[has])
    assert np.all(got[~has] == 0)
