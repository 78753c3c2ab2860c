"""The workspace's control words on the GPU, through the C ABI.

The layout's grid barrier counts arrivals in one of two counters, chosen by
the parity of `bar_gen`, and advances `bar_gen` once per call (zeroing the
other counter for the next call); the dispatch kernels hand out work by ticket
and the last CTA sets the tickets back to zero.  These tests check the words
themselves and the property they exist for: a workspace reused across calls of
different inputs - with a zero-token call, which skips the layout kernel and
clears the header on the host, in between - gives results bit-identical to the
oracle every time, and a second dispatch on a handle does all the work again.

Header words (int32 index): status 0, num_pad 1, pending 2, tok_ticket 3,
pad_ticket 4, done 5, bar_count 6 (even generations), bar_count_odd 7,
bar_gen 8.
"""
import ctypes

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


def _words(lay):
    torch.cuda.synchronize()
    return lay.workspace[:64].view(torch.int32).cpu().numpy()


def _rand(T, K, E, H, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int64)
    # skew: a few hot experts, so the per-chunk counts differ from seed to seed
    hot = rng.random((T, K)) < 0.3
    idx[hot] = rng.integers(0, 4, size=int(hot.sum()))     # repeats within a token are allowed
    w = rng.random((T, K)).astype(np.float32)
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    return idx, w, x


def test_reused_workspace_across_inputs_and_zero_token_calls(ep):
    """bar_gen advances by one per layout kernel; after each call the tickets
    and flags are back at zero, the counter of the call's parity holds its
    chunk count and the other is zero; a zero-token call in between
    (host-side clear, no kernel) keeps the next layout bit-exact."""
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    T, K, E, R, A, H = 4096, 8, 256, 8, 128, 256
    lay = ep.Layout(T, K, E, R, A, DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((11, 12, 13), start=1):
        idx, w, x = _rand(T, K, E, H, seed)
        lay = ep.layout(to_dev(idx), to_dev(w), E, R, A, out=lay)
        words = _words(lay)
        assert words[8] == call, "generation after call %d: %d" % (call, words[8])
        ref = oracle.layout(idx, w, E, R, A)
        check_layout(lay, ref)
        assert int(words[1]) == int(ref["off"][-1]) - int((idx >= 0).sum())   # num_pad
        assert (words[2:6] == 0).all()                    # pending, tickets
        assert words[6 + (call & 1)] == 0 and words[6 + ((call - 1) & 1)] > 0   # barrier counters
        # a call with no tokens on the same handle: counts and offsets zeroed, generation kept
        rc = lib.ep_layout(None, None, 0, K, E, R, A, 0, lay.ref(), stream)
        assert rc == 0
        words = _words(lay)
        assert words[8] == call and (words[:8] == 0).all()
        assert int(lay.expert_offset.abs().sum()) == 0
    assert ep.get_status(lay) == (ep.EP_OK, 0)


@pytest.mark.parametrize("fp8", [False, True])
def test_dispatch_tickets_reset(ep, fp8):
    """After every dispatch the ticket counters are zero again, so a second
    dispatch on the same handle does all the work and writes the same bytes."""
    cfg = workload.config("prefill_bf16")
    inp = workload.inputs(cfg)
    idx, w = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    x = to_dev_bf16(inp["x"])
    lay = ep.layout(idx, w, cfg["E"], cfg["R"], cfg["A"])
    first = ep.dispatch(lay, x, cast_to_fp8=fp8, do_zero_padding=True)
    words = _words(lay)
    assert (words[3], words[4], words[5]) == (0, 0, 0)
    if fp8:
        again = (torch.full_like(first[0].view(torch.uint8), 0x55).view(torch.float8_e4m3fn),
                 torch.full_like(first[1], 3.0))
        ep.dispatch(lay, x, cast_to_fp8=True, do_zero_padding=True, out=again[0], out_scales=again[1])
    else:
        again = torch.full_like(first.view(torch.int16), 0x5555).view(torch.bfloat16)
        ep.dispatch(lay, x, do_zero_padding=True, out=again)
    words = _words(lay)
    assert (words[3], words[4], words[5]) == (0, 0, 0)
    Np = lay.num_recv_rows()
    ref = oracle.layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"], cfg["A"])
    if fp8:
        rq, rs = oracle.cast_fp8(inp["x"])
        for got in (first, again):
            assert np.array_equal(fp8_bits(got[0][:Np]), oracle.dispatch_rows(rq, ref, True)[:Np])
            assert np.array_equal(f32_bits(got[1][:Np]), oracle.dispatch_rows(rs, ref, True)[:Np].view(np.uint32))
    else:
        exp = oracle.dispatch_rows(inp["x"], ref, True)[:Np]
        assert np.array_equal(bf16_bits(first[:Np]), exp)
        assert np.array_equal(bf16_bits(again[:Np]), exp)
    assert ep.get_status(lay) == (ep.EP_OK, 0)


def test_fused_call_advances_the_generation(ep):
    """ep_layout_dispatch runs the layout kernel and then the ticketed copy
    kernel (whose first row loads start while the layout runs): one
    generation per call, every ticket back at zero, the same bytes twice."""
    T, K, E, R, A, H = 2048, 8, 64, 4, 16, 512
    idx, w, x = _rand(T, K, E, H, 21)
    lay, recv = ep.layout_dispatch(to_dev(idx), to_dev(w), to_dev_bf16(x), E, R, A, do_zero_padding=True)
    assert _words(lay)[8] == 1
    ref = oracle.layout(idx, w, E, R, A)
    Np = check_layout(lay, ref)
    assert np.array_equal(bf16_bits(recv[:Np]), oracle.dispatch_rows(x, ref, True)[:Np])
    lay2, recv2 = ep.layout_dispatch(to_dev(idx), to_dev(w), to_dev_bf16(x), E, R, A, do_zero_padding=True,
                                     out_layout=lay, out=recv)
    assert _words(lay)[8] == 2 and (_words(lay)[2:6] == 0).all()
    assert np.array_equal(bf16_bits(recv2[:Np]), oracle.dispatch_rows(x, ref, True)[:Np])


def test_one_handle_across_batch_sizes(ep):
    """One workspace through layouts of different batch sizes, so the number of
    chunks (CTAs) changes from call to call while the two super-chunk sum
    buffers alternate with the generation: every call bit-exact."""
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    Tmax, K, E, R, A = 8192, 8, 256, 8, 128
    lay = ep.Layout(Tmax, K, E, R, A, DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, T in enumerate((8192, 640, 4096, 96, 8192, 1024, 2048), start=1):
        idx, w, _ = _rand(T, K, E, 8, 100 + call)
        d_idx, d_w = to_dev(idx), to_dev(w)
        rc = lib.ep_layout(ctypes.c_void_p(d_idx.data_ptr()), ctypes.c_void_p(d_w.data_ptr()), T, K, E, R, A, 0,
                           lay.ref(), stream)
        assert rc == 0
        torch.cuda.synchronize()
        ref = oracle.layout(idx, w, E, R, A)
        assert np.array_equal(lay.num_recv_tokens_per_expert.cpu().numpy(), ref["cnt"]), "call %d" % call
        assert np.array_equal(lay.expert_offset.cpu().numpy(), ref["off"]), "call %d" % call
        assert np.array_equal(lay._pair_slot_buf[:T * K].cpu().numpy(), ref["pair_slot"].reshape(-1))
        Np = int(ref["off"][-1])
        assert np.array_equal(lay.recv_src_token[:Np].cpu().numpy(), ref["recv_src"][:Np])
        assert _words(lay)[8] == call
    assert ep.get_status(lay) == (ep.EP_OK, 0)
