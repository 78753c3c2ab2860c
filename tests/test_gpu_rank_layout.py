"""The per-token-per-rank layout on the GPU against the oracle
("DeepEP 测试目标 API 系统性参考" §2.1 dispatch() without do_expand, §3.1
Buffer.dispatch() V1 layout quantities and receive outputs, §3.2
Buffer.combine(): the plain sum over the ranks a token reached).

Every output of ep_rank_layout bit-exact (is_token_in_rank, counts per rank
and expert, offsets, token slots, source tokens, local expert ids and
weights), then ep_dispatch (bf16 rows, the FP8 cast) and ep_combine on the
per-rank handle, over rank counts 1..32, -1 entries, alignment and weights;
the full prefill_bf16 workload; edge cases and error reporting."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import workload
from gpu_util import DEV, bf16_bits, f32_bits, fp8_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def check_rank_layout(lay, ref):
    rows = int(ref["rank_off"][-1])
    assert np.array_equal(lay.num_tokens_per_rank.cpu().numpy(), ref["num_tokens_per_rank"])
    assert np.array_equal(lay.rank_offset.cpu().numpy(), ref["rank_off"])
    assert np.array_equal(lay.is_token_in_rank.cpu().numpy(), ref["is_token_in_rank"])
    assert np.array_equal(lay.token_slot.cpu().numpy(), ref["token_slot"])
    assert np.array_equal(lay.num_tokens_per_expert.cpu().numpy(), ref["num_tokens_per_expert"])
    assert np.array_equal(lay.num_recv_tokens_per_expert.cpu().numpy(), ref["num_recv_tokens_per_expert"])
    assert np.array_equal(lay.recv_src_token[:rows].cpu().numpy(), ref["recv_src"][:rows])
    assert np.array_equal(lay.recv_topk_idx[:rows].cpu().numpy(), ref["recv_topk_idx"][:rows])
    assert np.array_equal(lay.recv_topk_weights[:rows].cpu().numpy().view(np.uint32),
                          ref["recv_topk_weights"][:rows].view(np.uint32))
    return rows


T, H, E, K = 320, 1152, 64, 6
MODES = list(itertools.product([1, 2, 8, 32], [0.0, 0.1], [True, False], [1, 128]))


@pytest.mark.parametrize("R,drop,weighted,A", MODES)
def test_rank_layout_modes(ep, R, drop, weighted, A):
    seed = hash((R, drop, weighted, A)) % (1 << 20)
    rng = np.random.default_rng(seed)
    scores = rng.standard_normal((T, E)) + np.linspace(0, 3, E)[None, :]
    idx = np.argsort(-scores, axis=1, kind="stable")[:, :K].astype(np.int64)
    if drop:
        idx[rng.random((T, K)) < drop] = -1
    w = rng.random((T, K)).astype(np.float32) if weighted else None
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    ref = oracle.rank_layout(idx, w, E, R, A)
    lay = ep.rank_layout(to_dev(idx), None if w is None else to_dev(w), E, R, A)
    recv = ep.dispatch(lay, to_dev_bf16(x))
    q, s = ep.dispatch(lay, to_dev_bf16(x), cast_to_fp8=True)
    rows = int(ref["rank_off"][-1])
    y = workload.expert_outputs(dict(seed=seed, H=H), max(rows, 1))
    nb = seed % 3
    biases = [workload.expert_outputs(dict(seed=seed, H=H), T, seed_offset=1 + i) for i in range(nb)]
    bias = None if nb == 0 else (to_dev_bf16(biases[0]) if nb == 1 else tuple(to_dev_bf16(b) for b in biases))
    out = ep.combine(lay, to_dev_bf16(y), bias=bias)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    check_rank_layout(lay, ref)
    assert np.array_equal(bf16_bits(recv[:rows]), oracle.dispatch_rows(x, ref, False)[:rows])
    rq, rs = oracle.cast_fp8(x)
    assert np.array_equal(fp8_bits(q[:rows]), oracle.dispatch_rows(rq, ref, False)[:rows])
    assert np.array_equal(f32_bits(s[:rows]), oracle.dispatch_rows(rs, ref, False)[:rows].view(np.uint32))
    exp = oracle.combine(y, ref["token_slot"], None, *(biases + [None] * (2 - nb)))
    assert np.array_equal(bf16_bits(out), exp)


def test_rank_layout_full_prefill(ep):
    cfg = workload.config("prefill_bf16")
    inp = workload.inputs(cfg)
    E_, R, A = cfg["E"], cfg["R"], cfg["A"]
    ref = oracle.rank_layout(inp["topk_idx"], inp["topk_weights"], E_, R, A)
    x = to_dev_bf16(inp["x"])
    lay = ep.rank_layout(to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), E_, R, A)
    recv = ep.dispatch(lay, x)
    rows = check_rank_layout(lay, ref)
    assert np.array_equal(bf16_bits(recv[:rows]), oracle.dispatch_rows(inp["x"], ref, False)[:rows])
    y = workload.expert_outputs(cfg, rows)
    out = ep.combine(lay, to_dev_bf16(y))
    assert np.array_equal(bf16_bits(out), oracle.combine(y, ref["token_slot"], None))
    assert ep.get_status(lay) == (ep.EP_OK, 0)


def test_rank_combine_reproduces_x(ep):
    """Expert outputs = x on each token's first rank, 0 elsewhere: combine gives x back."""
    cfg = workload.config("decode")
    inp = workload.inputs(cfg)
    lay = ep.rank_layout(to_dev(inp["topk_idx"]), None, cfg["E"], cfg["R"])
    x = to_dev_bf16(inp["x"])
    recv = ep.dispatch(lay, x)
    slot = lay.token_slot.long()
    first = torch.where(slot >= 0, torch.arange(cfg["R"], device=DEV)[None, :], cfg["R"]).min(dim=1).values
    keep = torch.zeros(lay.capacity, dtype=torch.bool, device=DEV)
    has = first < cfg["R"]
    keep[slot[has, first[has]]] = True
    y = torch.where(keep[:, None], recv, torch.zeros_like(recv))
    out = ep.combine(lay, y)
    got = bf16_bits(out)
    expect = np.where(inp["x"] == 0x8000, np.uint16(0), inp["x"])
    h = has.cpu().numpy()
    assert np.array_equal(got[h], expect[h]) and np.all(got[~h] == 0)


def test_rank_layout_edges(ep):
    # no tokens
    lay = ep.rank_layout(to_dev(np.zeros((0, 4), np.int64)), None, 16, 4)
    torch.cuda.synchronize()
    assert lay.rank_offset.cpu().tolist() == [0] * 5 and lay.num_tokens_per_expert.cpu().sum() == 0
    # every entry unselected; duplicates of one expert within a token; R = 1
    for idx in (-np.ones((8, 3), np.int64), np.tile(np.array([[5, 5, 1]], np.int64), (8, 1))):
        for R in (1, 4):
            ref = oracle.rank_layout(idx, None, 16, R, 4)
            lay = ep.rank_layout(to_dev(idx), None, 16, R, 4)
            torch.cuda.synchronize()
            check_rank_layout(lay, ref)
            assert ep.get_status(lay) == (ep.EP_OK, 0)


def test_rank_layout_errors(ep):
    idx = np.tile(np.array([[0, 3, 7]], np.int64), (16, 1))
    bad = idx.copy()
    bad[3, 1] = 99
    lay = ep.rank_layout(to_dev(bad), None, 8, 2)
    code, flags = ep.get_status(lay)
    assert code == ep.EP_ERR_BAD_EXPERT and flags & 1
    lay = ep.rank_layout(to_dev(idx), None, 8, 2, capacity=20)      # 32 rows needed
    code, flags = ep.get_status(lay)
    assert code == ep.EP_ERR_CAPACITY and flags & 2
    lay = ep.rank_layout(to_dev(idx), None, 8, 2)
    with pytest.raises(ep.EpError) as exc:
        ep.combine(lay, torch.zeros((32, 64), dtype=torch.bfloat16, device=DEV),
                   torch.ones((16, 3), dtype=torch.float32, device=DEV))
    assert exc.value.code == ep.EP_ERR_INVALID_ARG
    with pytest.raises(ep.EpError):
        ep.rank_layout(to_dev(np.zeros((64, 2), np.int64)), None, 64, 64)    # R above 32


def test_rank_layout_deterministic(ep):
    cfg = workload.config("prefill_bf16")
    inp = workload.inputs(cfg, with_x=False)
    idx, w = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    lay = ep.rank_layout(idx, w, cfg["E"], cfg["R"], cfg["A"])
    first = [t.clone() for t in (lay.token_slot, lay.recv_topk_idx, lay.recv_topk_weights, lay.recv_src_token)]
    for _ in range(10):
        ep.rank_layout(idx, w, cfg["E"], cfg["R"], cfg["A"], out=lay)
        for a, b in zip(first, (lay.token_slot, lay.recv_topk_idx, lay.recv_topk_weights, lay.recv_src_token)):
            assert torch.equal(a.view(torch.uint8) if a.dtype == torch.float32 else a,
                               b.view(torch.uint8) if b.dtype == torch.float32 else b)


@pytest.mark.parametrize("form", ["rank", "ll"])
def test_fp8_input_passthrough_other_forms(ep, form):
    """(e4m3 rows, fp32 scales) input is carried as is (§2.1: the received rows
    have the input's type) on the per-rank and fixed-slab handles too."""
    T, K, E, R, H = 96, 4, 32, 4, 512
    rng = np.random.default_rng(71)
    idx = rng.integers(-1, E, (T, K)).astype(np.int64)
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    q, s = oracle.cast_fp8(x)
    dq = torch.from_numpy(q).to(DEV).view(torch.float8_e4m3fn)
    ds = to_dev(s)
    if form == "rank":
        ref = oracle.rank_layout(idx, None, E, R)
        lay = ep.rank_layout(to_dev(idx), None, E, R)
    else:
        ref = oracle.ll_layout(idx, None, E, R, T // R + 1)
        lay = ep.ll_layout(to_dev(idx), None, E, R, T // R + 1)
    rq, rs = ep.dispatch(lay, dq, x_scales=ds, do_zero_padding=True)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    rows = int(ref["off"][-1])
    assert np.array_equal(fp8_bits(rq[:rows]), oracle.dispatch_rows(q, ref, True)[:rows])
    assert np.array_equal(f32_bits(rs[:rows]), oracle.dispatch_rows(s, ref, True)[:rows].view(np.uint32))
