"""Parity in the launch configuration the benchmark times: the step's calls
(layout, dispatch, combine) captured once as a CUDA graph (the programmatic
dependent-launch edges between the kernels kept) and replayed, at the full
prefill_bf16 and fp8_dispatch sizes, bit-exact against the oracle
("DeepEP 测试目标 API 系统性参考" §2.1, §2.2, §4.2); likewise the
per-token-per-rank step at prefill_bf16 (§3.1, §3.2) and the fixed-slab step
at the decode workload (§3.3, §3.4)."""
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


def _capture_and_replay(step, fill):
    """Warm once, capture the step as one graph, then replay it twice with the
    receive buffers overwritten and L2 flushed before each replay."""
    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=DEV)
    for _ in range(2):
        fill()
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()


def test_graph_replayed_per_rank_step_matches_oracle(ep):
    """The per-token-per-rank form as the benchmark's `--layout rank` step
    times it at prefill_bf16: ep_rank_layout, ep_dispatch and the plain
    (unweighted) sum over the reached ranks."""
    cfg = workload.config("prefill_bf16")
    inp = workload.inputs(cfg)
    E, R, A, T, K, H = cfg["E"], cfg["R"], cfg["A"], cfg["T"], cfg["K"], cfg["H"]
    ref = oracle.rank_layout(inp["topk_idx"], inp["topk_weights"], E, R, A)
    rows = int(ref["rank_off"][-1])
    y_host = workload.expert_outputs(cfg, rows)
    idx, w, x = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), to_dev_bf16(inp["x"])
    lay = ep.RankLayout(T, K, E, R, A, DEV)
    recv = torch.empty((lay.capacity, H), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((lay.capacity, H), dtype=torch.bfloat16, device=DEV)
    y[:rows] = to_dev_bf16(y_host)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)

    def step():
        ep.rank_layout(idx, w, E, R, A, out=lay)
        ep.dispatch(lay, x, do_zero_padding=cfg["zero_pad"], out=recv)
        ep.combine(lay, y, None, out=out)

    def fill():
        recv.view(torch.uint8).fill_(0xA5)
        lay.token_slot.fill_(-7)
        out.fill_(0)

    _capture_and_replay(step, fill)
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    assert np.array_equal(lay.token_slot.cpu().numpy(), ref["token_slot"])
    assert np.array_equal(lay.is_token_in_rank.cpu().numpy(), ref["is_token_in_rank"])
    assert np.array_equal(lay.num_recv_tokens_per_expert.cpu().numpy(), ref["num_recv_tokens_per_expert"])
    assert np.array_equal(lay.recv_topk_idx[:rows].cpu().numpy(), ref["recv_topk_idx"][:rows])
    assert np.array_equal(bf16_bits(recv[:rows]), oracle.dispatch_rows(inp["x"], ref, False)[:rows])
    assert np.array_equal(bf16_bits(out), oracle.combine(y_host, ref["token_slot"], None))


def test_graph_replayed_fixed_slab_step_matches_oracle(ep):
    """The fixed-slab form as the benchmark's `--layout ll` step times it at
    the decode workload (S = R * 128 rows per expert, 1 M receive rows, no
    zero padding), with identity experts (the receive buffer is the combine's
    input) and the weighted combine.  Only the pair rows are compared (the
    slab is 15 GB): each must hold its source token's row, and the combine
    is the oracle's over those rows."""
    cfg = workload.config("decode")
    inp = workload.inputs(cfg)
    E, R, T, H = cfg["E"], cfg["R"], cfg["T"], cfg["H"]
    M = cfg["max_tokens_per_rank"]
    ref = oracle.ll_layout(inp["topk_idx"], inp["topk_weights"], E, R, M)
    idx, w, x = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), to_dev_bf16(inp["x"])
    lay = ep.ll_layout(idx, w, E, R, M)
    recv = torch.empty((lay.capacity, H), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)

    def step():
        ep.ll_layout(idx, w, E, R, M, out=lay)
        ep.dispatch(lay, x, do_zero_padding=cfg["zero_pad"], out=recv)
        ep.combine(lay, recv, w, out=out)

    def fill():
        recv[:: 4096].view(torch.uint8).fill_(0xA5)      # one row in 4096 (the slab is 15 GB)
        lay.pair_slot.fill_(-7)
        out.fill_(0)

    _capture_and_replay(step, fill)
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    assert np.array_equal(lay.pair_slot.cpu().numpy(), ref["pair_slot"])
    assert np.array_equal(lay.expert_offset.cpu().numpy(), ref["off"])
    assert np.array_equal(lay.recv_src_token.cpu().numpy(), ref["recv_src"])
    sel = np.nonzero(ref["recv_src"] >= 0)[0]
    got = bf16_bits(recv.index_select(0, torch.from_numpy(sel).to(DEV)))
    assert np.array_equal(got, inp["x"][ref["recv_src"][sel]])
    # the combine reads only pair rows: renumber them densely for the oracle
    dense = np.full(lay.capacity, -1, np.int64)
    dense[sel] = np.arange(sel.size)
    ps = ref["pair_slot"]
    slot_c = np.where(ps >= 0, dense[np.maximum(ps, 0)], -1).astype(ps.dtype)
    assert np.array_equal(bf16_bits(out), oracle.combine(got, slot_c, inp["topk_weights"]))
