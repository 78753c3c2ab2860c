"""Dispatch and combine over receive regions held as separate buffers, filled
by several source groups, on one GPU (the one-GPU part of expert parallelism
over several GPUs; §2.1 dispatch() / §2.2 combine() across ranks).

The batch is split into G source groups; each runs ep_layout (alignment 1) on
its tokens, the groups' counts are gathered, and each group dispatches its
rows into R region buffers allocated separately (on several GPUs they would be
peer memory).  The regions must then hold, byte for byte, the rows of the
oracle's layout of the concatenated batch, region r being its rows
[off[r*E/R], off[(r+1)*E/R]) with zero padding; combine from the regions must
give each group's tokens the oracle's combine bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import workload
from gpu_util import DEV, bf16_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def _run(ep, name, G, pad_on_last=True):
    cfg = workload.config(name)
    inp = workload.inputs(cfg)
    T, H, E, R, A = cfg["T"], cfg["H"], cfg["E"], cfg["R"], cfg["A"]
    El = E // R
    Tg = T // G
    idx_h, w_h, x_h = inp["topk_idx"], inp["topk_weights"], inp["x"]
    ref = oracle.layout(idx_h, w_h, E, R, A)
    off = ref["off"].astype(np.int64)
    # every group's own layout, then the count exchange
    groups = []
    for g in range(G):
        sl = slice(g * Tg, (g + 1) * Tg)
        idx, w, x = to_dev(idx_h[sl]), to_dev(w_h[sl]), to_dev_bf16(x_h[sl])
        lay = ep.layout(idx, w, E, R, 1)
        groups.append((sl, idx, w, x, lay))
    counts = np.stack([lay.num_recv_tokens_per_expert.cpu().numpy() for (_, _, _, _, lay) in groups])
    assert np.array_equal(counts.sum(0), ref["cnt"])
    offs = [ep.source_offsets(counts, R, A, g) for g in range(G)]
    rows = offs[0][1]
    cap = int(rows.max()) + 3
    regions = [torch.full((cap, H), -1.0, dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    table = ep.RegionTable(regions)          # built once, used by every group's call
    for g, (sl, idx, w, x, lay) in enumerate(groups):
        delta, rows_g, pads = offs[g]
        assert np.array_equal(rows_g, rows)
        last = g == G - 1
        ep.dispatch_regions(lay, idx, to_dev(delta), table, x,
                            pad_list=to_dev(pads) if (last and pad_on_last and len(pads)) else None)
    torch.cuda.synchronize()
    exp = oracle.dispatch_rows(x_h, ref, True)
    for r in range(R):
        lo, hi = int(off[r * El]), int(off[(r + 1) * El])
        assert rows[r] == hi - lo
        assert np.array_equal(bf16_bits(regions[r][:hi - lo]), exp[lo:hi]), "region %d" % r
        # nothing past the region's rows was touched
        assert bool((regions[r][hi - lo:] == -1.0).all())
    for (_, _, _, _, lay) in groups:
        assert ep.get_status(lay) == (ep.EP_OK, 0)
        assert (lay.workspace[12:24].view(torch.int32) == 0).all()      # tickets reset
    # combine: expert outputs in the concatenated receive order, split into regions
    Np = int(off[-1])
    y = workload.expert_outputs(cfg, Np)
    yreg = [torch.zeros((cap, H), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    for r in range(R):
        lo, hi = int(off[r * El]), int(off[(r + 1) * El])
        yreg[r][:hi - lo] = to_dev_bf16(y[lo:hi])
    for g, (sl, idx, w, x, lay) in enumerate(groups):
        out = ep.combine_regions(lay, idx, to_dev(offs[g][0]), yreg, w)
        want = oracle.combine(y, ref["pair_slot"][sl], w_h[sl])
        assert np.array_equal(bf16_bits(out), want), "group %d" % g


@pytest.mark.parametrize("name,G", [("prefill_bf16", 2), ("prefill_bf16", 4), ("decode", 2),
                                    ("large_prefill", 4), ("tiny", 2)])
def test_regions_match_the_concatenated_layout(ep, name, G):
    _run(ep, name, G)


def test_regions_reject_an_aligned_handle(ep):
    cfg = workload.config("tiny")
    inp = workload.inputs(cfg)
    idx = to_dev(inp["topk_idx"])
    lay = ep.layout(idx, None, cfg["E"], cfg["R"], 4)          # alignment 4: not a group layout
    regions = [torch.zeros((64, cfg["H"]), dtype=torch.bfloat16, device=DEV) for _ in range(cfg["R"])]
    delta = torch.zeros(cfg["E"], dtype=torch.int32, device=DEV)
    with pytest.raises(ep.EpError):
        ep.dispatch_regions(lay, idx, delta, regions, to_dev_bf16(inp["x"]))


def test_regions_with_two_segment_rows(ep):
    """bf16 rows of 32 KB (H = 16384) travel as two bulk segments; padding
    rows are zeroed in 2 KB pieces; G = 3 groups of ragged sizes."""
    rng = np.random.default_rng(5)
    T, K, E, R, A, H = 96, 4, 16, 4, 8, 16384
    idx_h = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int64)
    idx_h[rng.random(idx_h.shape) < 0.15] = -1
    w_h = rng.random((T, K)).astype(np.float32)
    x_h = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    ref = oracle.layout(idx_h, w_h, E, R, A)
    off = ref["off"].astype(np.int64)
    El = E // R
    cuts = [0, 40, 44, 96]                     # groups of 40, 4 and 52 tokens
    groups = []
    for g in range(3):
        sl = slice(cuts[g], cuts[g + 1])
        idx, w = to_dev(idx_h[sl]), to_dev(w_h[sl])
        groups.append((sl, idx, w, to_dev_bf16(x_h[sl]), ep.layout(idx, w, E, R, 1)))
    counts = np.stack([lay.num_recv_tokens_per_expert.cpu().numpy() for (_, _, _, _, lay) in groups])
    offs = [ep.source_offsets(counts, R, A, g) for g in range(3)]
    cap = int(offs[0][1].max())
    regions = [torch.full((cap, H), 7.0, dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    for g, (sl, idx, w, x, lay) in enumerate(groups):
        pads = offs[g][2]
        ep.dispatch_regions(lay, idx, to_dev(offs[g][0]), regions, x, pad_list=to_dev(pads) if g == 0 else None)
    torch.cuda.synchronize()
    exp = oracle.dispatch_rows(x_h, ref, True)
    for r in range(R):
        lo, hi = int(off[r * El]), int(off[(r + 1) * El])
        assert np.array_equal(bf16_bits(regions[r][:hi - lo]), exp[lo:hi]), "region %d" % r
    y = workload.expert_outputs(dict(seed=9, H=H), int(off[-1]))
    yreg = [torch.zeros((cap, H), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    for r in range(R):
        lo, hi = int(off[r * El]), int(off[(r + 1) * El])
        yreg[r][:hi - lo] = to_dev_bf16(y[lo:hi])
    for g, (sl, idx, w, x, lay) in enumerate(groups):
        out = ep.combine_regions(lay, idx, to_dev(offs[g][0]), yreg, w)
        assert np.array_equal(bf16_bits(out), oracle.combine(y, ref["pair_slot"][sl], w_h[sl]))
