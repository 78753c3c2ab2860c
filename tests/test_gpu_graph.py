"""Parity in the launch configuration the benchmark times: the step's calls
(layout, dispatch, combine) captured once as a CUDA graph (the programmatic
dependent-launch edges between the kernels kept) and replayed, at the full
prefill_bf16 and fp8_dispatch sizes, bit-exact against the oracle
("DeepEP 测试目标 API 系统性参考" §2.1, §2.2, §4.2)."""
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


@pytest.mark.parametrize("name", ["prefill_bf16", "fp8_dispatch"])
def test_graph_replayed_step_matches_oracle(ep, name):
    cfg = workload.config(name)
    inp = workload.inputs(cfg)
    E, R, A, T, H = cfg["E"], cfg["R"], cfg["A"], cfg["T"], cfg["H"]
    ref = oracle.layout(inp["topk_idx"], inp["topk_weights"], E, R, A)
    Np = int(ref["off"][-1])
    y_host = workload.expert_outputs(cfg, Np)
    idx, w, x = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), to_dev_bf16(inp["x"])
    lay = ep.Layout(T, cfg["K"], E, R, A, DEV)
    y = torch.zeros((lay.capacity, H), dtype=torch.bfloat16, device=DEV)
    y[:Np] = to_dev_bf16(y_host)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    if cfg["fp8"]:
        recv = torch.empty((lay.capacity, H), dtype=torch.float8_e4m3fn, device=DEV)
        scales = torch.empty((lay.capacity, H // 128), dtype=torch.float32, device=DEV)
    else:
        recv = torch.empty((lay.capacity, H), dtype=torch.bfloat16, device=DEV)
        scales = None

    def step():
        ep.layout(idx, w, E, R, A, out=lay)
        if cfg["fp8"]:
            ep.dispatch(lay, x, cast_to_fp8=True, do_zero_padding=True, out=recv, out_scales=scales)
        else:
            ep.dispatch(lay, x, do_zero_padding=cfg["zero_pad"], out=recv)
        ep.combine(lay, y, w, out=out)

    step()                                   # warm (and sizes every launch) before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=DEV)
    for _ in range(2):
        recv.view(torch.uint8).fill_(0xA5)   # stale bytes everywhere before each replay
        out.fill_(0)
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    check_layout(lay, ref)
    if cfg["fp8"]:
        rq, rs = oracle.cast_fp8(inp["x"])
        assert np.array_equal(fp8_bits(recv[:Np]), oracle.dispatch_rows(rq, ref, True)[:Np])
        assert np.array_equal(f32_bits(scales[:Np]), oracle.dispatch_rows(rs, ref, True)[:Np].view(np.uint32))
    else:
        assert np.array_equal(bf16_bits(recv[:Np]), oracle.dispatch_rows(inp["x"], ref, cfg["zero_pad"])[:Np])
    assert np.array_equal(bf16_bits(out), oracle.combine(y_host, ref["pair_slot"], inp["topk_weights"]))
