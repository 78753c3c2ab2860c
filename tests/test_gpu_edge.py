"""Edge cases, device-side error reporting, determinism and batch invariance
on the GPU, through the C ABI.

Error reporting follows the library's contract: bad expert ids and receive
overflow are reported in the device status word, never by a fault; every wait
is bounded (the self-test makes one run out on purpose and checks the status).
Batch invariance follows the pattern of the SGLang DeepGEMM batch-invariance
test (rows of a batch computed alone and inside larger batches must match with
atol = rtol = 0).
"""
import hashlib

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


def _full(ep, idx, w, x, E, R, A, zero_pad=True, fp8=False, fused=False):
    ref = oracle.layout(idx, w, E, R, A)
    xd = to_dev_bf16(x)
    if fused:
        lay, res = ep.layout_dispatch(to_dev(idx), None if w is None else to_dev(w), xd, E, R, A,
                                      cast_to_fp8=fp8, do_zero_padding=zero_pad)
    else:
        lay = ep.layout(to_dev(idx), None if w is None else to_dev(w), E, R, A)
        res = ep.dispatch(lay, xd, cast_to_fp8=fp8, do_zero_padding=zero_pad)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    Np = check_layout(lay, ref)
    if fp8:
        rq, rs = oracle.cast_fp8(x)
        assert np.array_equal(fp8_bits(res[0][:Np]), oracle.dispatch_rows(rq, ref, zero_pad)[:Np])
        assert np.array_equal(f32_bits(res[1][:Np]), oracle.dispatch_rows(rs, ref, zero_pad)[:Np].view(np.uint32))
    else:
        assert np.array_equal(bf16_bits(res[:Np]), oracle.dispatch_rows(x, ref, zero_pad)[:Np])
    if Np:
        y = workload.expert_outputs(dict(seed=5, H=x.shape[1]), Np)
        out = ep.combine(lay, to_dev_bf16(y), None if w is None else to_dev(w))
        assert np.array_equal(bf16_bits(out), oracle.combine(y, ref["pair_slot"], w))
    return lay, ref


def _rand(T, K, E, H, seed=0, drop=0.0):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int64).reshape(T, K)
    if drop:
        idx[rng.random((T, K)) < drop] = -1
    w = rng.random((T, K)).astype(np.float32)
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    return idx, w, x


def test_zero_tokens(ep):
    idx = np.zeros((0, 4), np.int64)
    lay = ep.layout(to_dev(idx), None, 16, 2, 4)
    recv = ep.dispatch(lay, torch.zeros((0, 256), dtype=torch.bfloat16, device=DEV), do_zero_padding=True)
    out = ep.combine(lay, torch.zeros((4, 256), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert out.shape == (0, 256) and recv.shape[1] == 256
    assert lay.expert_offset.cpu().tolist() == [0] * 17
    assert ep.get_status(lay) == (ep.EP_OK, 0)


def test_all_unselected(ep):
    T, K, E, H = 64, 4, 16, 256
    idx = -np.ones((T, K), np.int64)
    _, w, x = _rand(T, K, E, H)
    lay, ref = _full(ep, idx, w, x, E, 2, 8)
    out = ep.combine(lay, torch.zeros((1, H), dtype=torch.bfloat16, device=DEV), to_dev(w))
    assert np.all(bf16_bits(out) == 0)


@pytest.mark.parametrize("T,K,E,R,A,H", [
    (1, 1, 1, 1, 1, 8),            # smallest everything
    (1, 8, 256, 1, 128, 7168),     # single token
    (7, 3, 12, 1, 5, 24),          # ragged everything, H = 24 (48-byte rows)
    (96, 32, 64, 4, 3, 136),       # K = 32 (the maximum), H = 136
    (130, 2, 4, 2, 128, 4096),     # few experts, heavy padding
    (256, 8, 4096, 4, 1, 512),     # E at the maximum
    (64, 4, 16, 16, 2, 16384),     # bf16 rows of 32 KB: two bulk segments per row
    (4099, 8, 256, 1, 7, 7168),    # ragged chunking of a larger batch
])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_shapes_bf16(ep, T, K, E, R, A, H, fused):
    idx, w, x = _rand(T, K, E, H, seed=T + K, drop=0.1)
    _full(ep, idx, w, x, E, R, A, fused=fused)


@pytest.mark.parametrize("T,K,E,R,A,H", [
    (5, 2, 8, 1, 4, 128),          # one scale per row (4-byte scale rows, plain stores)
    (33, 8, 32, 1, 16, 640),       # 5 scales per row
    (64, 4, 16, 2, 1, 16384),      # the largest row the cast kernel stages
])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_shapes_fp8(ep, T, K, E, R, A, H, fused):
    idx, w, x = _rand(T, K, E, H, seed=3 * T + K, drop=0.1)
    _full(ep, idx, w, x, E, R, A, fp8=True, fused=fused)


@pytest.mark.parametrize("H", [1024, 640, 128], ids=["sf32B", "sf20B", "sf4B"])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_fp8_input_passthrough(ep, fused, H):
    """(e4m3, scales) input is dispatched as is: rows and scale rows move together.
    The padding rows' scales are zeroed by a bulk store when the scale row is a
    multiple of 16 bytes (H = 1024: 32 B), else by plain stores (20 B, 4 B)."""
    T, K, E, R, A = 200, 8, 64, 4, 16
    idx, w, x = _rand(T, K, E, H, seed=11)
    q, s = oracle.cast_fp8(x)
    ref = oracle.layout(idx, w, E, R, A)
    xq = to_dev(q).view(torch.float8_e4m3fn)
    if fused:
        lay, (rq, rs) = ep.layout_dispatch(to_dev(idx), to_dev(w), xq, E, R, A, x_scales=to_dev(s),
                                           do_zero_padding=True)
    else:
        lay = ep.layout(to_dev(idx), to_dev(w), E, R, A)
        rq, rs = ep.dispatch(lay, xq, x_scales=to_dev(s), do_zero_padding=True)
    Np = int(ref["off"][-1])
    assert np.array_equal(fp8_bits(rq[:Np]), oracle.dispatch_rows(q, ref, True)[:Np])
    assert np.array_equal(f32_bits(rs[:Np]), oracle.dispatch_rows(s, ref, True)[:Np].view(np.uint32))


def test_standalone_cast(ep):
    x = np.concatenate([workload.tokens(workload.config("prefill_bf16"), rows=300),
                        np.zeros((1, 7168), np.uint16)])
    q, s = ep.cast_fp8(to_dev_bf16(x))
    rq, rs = oracle.cast_fp8(x)
    assert np.array_equal(fp8_bits(q), rq)
    assert np.array_equal(f32_bits(s), rs.view(np.uint32))


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_bad_expert_reported(ep, fused):
    T, K, E, H = 32, 4, 16, 256
    idx, w, x = _rand(T, K, E, H)
    idx[3, 1] = E
    idx[7, 0] = -5
    if fused:
        lay, _ = ep.layout_dispatch(to_dev(idx), to_dev(w), to_dev_bf16(x), E, 2, 1)
    else:
        lay = ep.layout(to_dev(idx), to_dev(w), E, 2, 1)
        ep.dispatch(lay, to_dev_bf16(x))
    code, flags = ep.get_status(lay)
    assert code == ep.EP_ERR_BAD_EXPERT and flags & 1
    # the bad entries are treated as unselected
    ps = lay.pair_slot.cpu().numpy()
    assert ps[3, 1] == -1 and ps[7, 0] == -1
    # a later good layout on the same handle clears the status
    idx2 = np.where(idx >= E, 0, np.maximum(idx, -1))
    ep.layout(to_dev(idx2), to_dev(w), E, 2, 1, out=lay)
    assert ep.get_status(lay) == (ep.EP_OK, 0)


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_capacity_overflow_reported(ep, fused):
    T, K, E, H, A = 64, 4, 16, 256, 8
    idx, w, x = _rand(T, K, E, H)
    if fused:
        lay, recv = ep.layout_dispatch(to_dev(idx), to_dev(w), to_dev_bf16(x), E, 2, A, capacity=100,
                                       do_zero_padding=True)
    else:
        lay = ep.layout(to_dev(idx), to_dev(w), E, 2, A, capacity=100)
        recv = ep.dispatch(lay, to_dev_bf16(x), do_zero_padding=True)
    ep.combine(lay, recv, to_dev(w))
    code, flags = ep.get_status(lay)
    assert code == ep.EP_ERR_CAPACITY and flags & 2


def test_tokens_per_rank_limit(ep):
    idx = np.zeros((256, 2), np.int64)
    with pytest.raises(ep.EpError) as exc:
        ep.layout(to_dev(idx), None, 8, 2, 1, num_max_tokens_per_rank=127)
    assert exc.value.code == ep.EP_ERR_CAPACITY
    ep.layout(to_dev(idx), None, 8, 2, 1, num_max_tokens_per_rank=128)


def test_invalid_arguments(ep):
    idx = to_dev(np.zeros((8, 2), np.int64))
    for args in [(8, 3, 1), (8, 2, 0), (8, 0, 1)]:
        with pytest.raises(ep.EpError) as exc:
            ep.layout(idx, None, *args)
        assert exc.value.code == ep.EP_ERR_INVALID_ARG
    lay = ep.layout(idx, None, 8, 2, 1)
    with pytest.raises(ep.EpError):   # H % 128 != 0 with the FP8 cast
        ep.dispatch(lay, torch.zeros((8, 136), dtype=torch.bfloat16, device=DEV), cast_to_fp8=True)


def test_bounded_wait_selftest(ep):
    idx, w, x = _rand(16, 2, 8, 64)
    lay = ep.layout(to_dev(idx), to_dev(w), 8, 2, 1)
    ep.selftest_bounded_wait(lay, 2_000_000)       # 2 ms on a barrier nothing completes
    code, flags = ep.get_status(lay)
    assert code == ep.EP_ERR_TIMEOUT and flags & 4
    _full(ep, idx, w, x, 8, 2, 1)                  # the context is still usable


def _hash(*ts):
    h = hashlib.sha256()
    for t in ts:
        h.update(t.contiguous().view(torch.uint8).cpu().numpy().tobytes())
    return h.hexdigest()


def test_determinism_repeated_runs(ep):
    cfg = workload.config("prefill_bf16")
    inp = workload.inputs(cfg)
    idx, w, x = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), to_dev_bf16(inp["x"])
    seen = set()
    for _ in range(20):
        lay = ep.layout(idx, w, cfg["E"], cfg["R"], cfg["A"])
        recv = ep.dispatch(lay, x, do_zero_padding=True)
        out = ep.combine(lay, recv, w)
        Np = lay.num_recv_rows()
        seen.add(_hash(lay.pair_slot, lay.recv_src_token[:Np], recv[:Np], out))
    assert len(seen) == 1


def test_batch_invariance(ep):
    """Rows of the first tokens are identical whether combined in a batch of
    1, 16, 64 or 257 tokens (the layout, and so every slot, changes with B)."""
    T, K, E, H = 257, 8, 64, 512
    idx, w, x = _rand(T, K, E, H, seed=21, drop=0.05)
    outs = {}
    for B in (1, 16, 64, 257):
        lay = ep.layout(to_dev(idx[:B]), to_dev(w[:B]), E, 1, 4)
        recv = ep.dispatch(lay, to_dev_bf16(x[:B]), do_zero_padding=True)
        # a per-expert transform stands in for the experts: y = recv * (1 + lexp / 64)
        scale = 1.0 + lay.recv_local_expert.clamp(min=0).float() / 64.0
        y = (recv.float() * scale[:recv.shape[0], None]).to(torch.bfloat16)
        outs[B] = bf16_bits(ep.combine(lay, y, to_dev(w[:B])))
    for B in (16, 64, 257):
        assert np.array_equal(outs[B][:1], outs[1])
    assert np.array_equal(outs[257][:16], outs[16]) and np.array_equal(outs[257][:64], outs[64])


def test_recv_stats_accumulate_over_calls(ep):
    """cumulative_local_expert_recv_stats (§2.1, §3.3): each layout adds its
    per-expert counts; a call without the tensor, or with no tokens, adds nothing."""
    T, K, E, R, A, H = 256, 8, 64, 4, 8, 128
    stats0 = np.arange(E, dtype=np.int32) * 1000
    stats = to_dev(stats0)
    expect = stats0
    lay = None
    for seed in (1, 2, 3):
        idx, w, x = _rand(T, K, E, H, seed=seed, drop=0.1)
        ref = oracle.layout(idx, w, E, R, A)
        lay = ep.layout(to_dev(idx), to_dev(w), E, R, A, out=lay, cumulative_local_expert_recv_stats=stats)
        expect = oracle.accumulate_recv_stats(expect, ref["cnt"])
    lay, _ = ep.layout_dispatch(to_dev(idx), to_dev(w), to_dev_bf16(x), E, R, A, out_layout=lay,
                                cumulative_local_expert_recv_stats=stats)
    expect = oracle.accumulate_recv_stats(expect, ref["cnt"])
    ep.layout(to_dev(idx), to_dev(w), E, R, A, out=lay)                     # no stats: unchanged
    ep.layout(to_dev(np.zeros((0, K), np.int64)), None, E, R, A, cumulative_local_expert_recv_stats=stats)
    torch.cuda.synchronize()
    assert np.array_equal(stats.cpu().numpy(), expect)


@pytest.mark.parametrize("T,K,E,H,num_bias", [(64, 4, 16, 24, 1), (64, 4, 16, 24, 2), (33, 32, 64, 1032, 2),
                                              (5, 1, 4, 8, 1)])
def test_combine_bias_shapes(ep, T, K, E, H, num_bias):
    """Bias with ragged rows (H = 24, 1032: rows not a multiple of the 2 KB item),
    K at its maximum, all-unselected tokens (out = bf16(bias0 [+ bias1]))."""
    idx, w, _ = _rand(T, K, E, H, seed=T * K, drop=0.2)
    idx[:3] = -1
    lay = ep.layout(to_dev(idx), to_dev(w), E, 1, 2)
    ref = oracle.layout(idx, w, E, 1, 2)
    Np = int(ref["off"][-1])
    cfg = dict(seed=T + K + H, H=H)
    y = workload.expert_outputs(cfg, max(Np, 1))
    biases = [workload.expert_outputs(cfg, T, seed_offset=1 + i) for i in range(num_bias)]
    dev_b = [to_dev_bf16(b) for b in biases]
    out = ep.combine(lay, to_dev_bf16(y), to_dev(w), bias=dev_b[0] if num_bias == 1 else tuple(dev_b))
    exp = oracle.combine(y, ref["pair_slot"], w, *(biases + [None] * (2 - num_bias)))
    assert np.array_equal(bf16_bits(out), exp)


def test_combine_in_place_over_bias(ep):
    """out may be bias0 itself: every element reads its bias before it is written."""
    T, K, E, H = 128, 8, 32, 7168
    idx, w, _ = _rand(T, K, E, H, seed=5, drop=0.1)
    lay = ep.layout(to_dev(idx), to_dev(w), E, 2, 1)
    ref = oracle.layout(idx, w, E, 2, 1)
    cfg = dict(seed=77, H=H)
    y = workload.expert_outputs(cfg, int(ref["off"][-1]))
    b0 = workload.expert_outputs(cfg, T, seed_offset=1)
    d_b0 = to_dev_bf16(b0)
    out = ep.combine(lay, to_dev_bf16(y), to_dev(w), bias=d_b0, out=d_b0)
    assert out.data_ptr() == d_b0.data_ptr()
    assert np.array_equal(bf16_bits(out), oracle.combine(y, ref["pair_slot"], w, b0, None))


def test_combine_second_bias_alone_rejected(ep):
    idx, w, _ = _rand(16, 2, 8, 64)
    lay = ep.layout(to_dev(idx), to_dev(w), 8, 2, 1)
    b = torch.zeros((16, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ep.EpError) as exc:
        ep.combine(lay, torch.zeros((64, 64), dtype=torch.bfloat16, device=DEV), bias=(None, b))
    assert exc.value.code == ep.EP_ERR_INVALID_ARG


@pytest.mark.parametrize("form", ["expand", "rank"])
def test_layout_many_rounds_per_warp(ep, form):
    """More than four rounds of 32 pairs per warp (over 2048 pairs per chunk at
    the 128-chunk limit), so the assign pass reloads keys beyond the ones it
    keeps in registers: 65536 tokens x top-8 (524 k pairs), skewed experts."""
    cfg = dict(workload.config("prefill_bf16"), T=65536)
    idx, w = workload.routing(cfg)
    E, R, A = cfg["E"], cfg["R"], cfg["A"]
    if form == "expand":
        ref = oracle.layout(idx, w, E, R, A)
        lay = ep.layout(to_dev(idx), to_dev(w), E, R, A)
        torch.cuda.synchronize()
        assert ep.get_status(lay) == (ep.EP_OK, 0)
        check_layout(lay, ref)
    else:
        ref = oracle.rank_layout(idx, w, E, R, A)
        lay = ep.rank_layout(to_dev(idx), to_dev(w), E, R, A)
        torch.cuda.synchronize()
        assert ep.get_status(lay) == (ep.EP_OK, 0)
        rows = int(ref["rank_off"][-1])
        assert np.array_equal(lay.token_slot.cpu().numpy(), ref["token_slot"])
        assert np.array_equal(lay.recv_src_token[:rows].cpu().numpy(), ref["recv_src"][:rows])
        assert np.array_equal(lay.recv_topk_idx[:rows].cpu().numpy(), ref["recv_topk_idx"][:rows])
        assert np.array_equal(lay.num_tokens_per_expert.cpu().numpy(), ref["num_tokens_per_expert"])


def test_fused_layout_dispatch_many_rounds(ep):
    """ep_layout_dispatch (one CTA per SM) at 65536 tokens x top-8: about 220
    pairs per warp, so its layout pass reloads keys too; 512-byte rows."""
    cfg = dict(workload.config("prefill_bf16"), T=65536, H=256)
    idx, w = workload.routing(cfg)
    x = workload.tokens(cfg)
    E, R, A = cfg["E"], cfg["R"], cfg["A"]
    ref = oracle.layout(idx, w, E, R, A)
    lay, recv = ep.layout_dispatch(to_dev(idx), to_dev(w), to_dev_bf16(x), E, R, A, do_zero_padding=True)
    torch.cuda.synchronize()
    assert ep.get_status(lay) == (ep.EP_OK, 0)
    Np = check_layout(lay, ref)
    assert np.array_equal(bf16_bits(recv[:Np]), oracle.dispatch_rows(x, ref, True)[:Np])


def _copy_grid():
    """CTAs of the copy kernel: four per SM (its three 16 KB stages fit four times)."""
    return 4 * torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("dT", [-3, 0, 5])
@pytest.mark.parametrize("H", [16384, 7168], ids=["row32KB", "row14KB"])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_tail_segments_around_the_split(ep, dT, H, fused):
    """Without padding that could fill the tail (A = 1) the copy kernel hands
    out the last 2 x grid tokens as segments of at most 4 KB.  Batches just
    below, at and above that many tokens (all tokens small, none but a few
    large) with rows of one and two 16 KB segments: bit-exact rows and
    combine."""
    T = 2 * _copy_grid() + dT
    T -= T % 4
    idx, w, x = _rand(T, 6, 64, H, seed=T + H, drop=0.05)
    _full(ep, idx, w, x, 64, 4, 1, fused=fused)


def test_tail_segments_fp8_input(ep):
    """e4m3 rows (7 KB: one segment, two in the tail) with their scale rows,
    carried once per token from the first segment."""
    T, K, E, R, A, H = 2 * _copy_grid() + 8, 8, 64, 4, 1, 7168
    idx, w, x = _rand(T, K, E, H, seed=3)
    q, s = oracle.cast_fp8(x)
    ref = oracle.layout(idx, w, E, R, A)
    lay = ep.layout(to_dev(idx), to_dev(w), E, R, A)
    rq, rs = ep.dispatch(lay, to_dev(q).view(torch.float8_e4m3fn), x_scales=to_dev(s), do_zero_padding=True)
    torch.cuda.synchronize()
    Np = int(ref["off"][-1])
    assert np.array_equal(fp8_bits(rq[:Np]), oracle.dispatch_rows(q, ref, True)[:Np])
    assert np.array_equal(f32_bits(rs[:Np]), oracle.dispatch_rows(s, ref, True)[:Np].view(np.uint32))
