"""ep_layout_no_alloc, the layout entry point for callers that cannot allocate
device memory themselves (a plain C host program with no device allocator of
its own, or a process whose device memory belongs to another framework's
pool): its workspace is a fixed array in the library's own device memory.

Through the C ABI, two calls in a row (different workloads, so stale contents
of the shared array would show) must give the same bytes as ep_layout with a
caller-owned workspace, and a dispatch on the returned handle must match too.
A call the argument checks reject must leave the shared array untouched; a
call with no tokens gives zero counts; an older handle stays valid for an
unpadded dispatch and for combine after a newer call.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import workload
from gpu_util import DEV, bf16_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def _handle(cfg, dev):
    """A handle whose arrays the test allocates; no workspace is given."""
    from combine_ep_layout_11_b200 import _lib
    T, K, E, A = cfg["T"], cfg["K"], cfg["E"], cfg["A"]
    cap = T * K + E * (A - 1)
    arrs = dict(cnt=torch.empty(E, dtype=torch.int32, device=dev),
                off=torch.empty(E + 1, dtype=torch.int32, device=dev),
                pair_slot=torch.empty(max(T * K, 1), dtype=torch.int32, device=dev),
                recv_src=torch.empty(cap, dtype=torch.int32, device=dev),
                recv_w=torch.empty(cap, dtype=torch.float32, device=dev),
                recv_lexp=torch.empty(cap, dtype=torch.int32, device=dev))
    s = _lib.EpLayout()
    s.num_recv_tokens_per_expert = arrs["cnt"].data_ptr()
    s.expert_offset = arrs["off"].data_ptr()
    s.pair_slot = arrs["pair_slot"].data_ptr()
    s.recv_src_token = arrs["recv_src"].data_ptr()
    s.recv_weight = arrs["recv_w"].data_ptr()
    s.recv_local_expert = arrs["recv_lexp"].data_ptr()
    s.workspace = None
    s.workspace_bytes = 0
    s.capacity = cap
    return s, arrs


def test_no_alloc_layout_matches_ep_layout_twice(ep):
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for name in ("prefill_bf16", "decode"):          # two calls in a row
        cfg = workload.config(name)
        inp = workload.inputs(cfg)
        idx, w = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
        x = to_dev_bf16(inp["x"])
        ref = ep.layout(idx, w, cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"])
        ref_recv = ep.dispatch(ref, x, do_zero_padding=cfg["zero_pad"])

        s, arrs = _handle(cfg, DEV)
        rc = lib.ep_layout_no_alloc(ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                    cfg["T"], cfg["K"], cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"],
                                    ctypes.byref(s), stream)
        assert rc == 0, lib.ep_status_string(rc)
        assert s.workspace and s.workspace_bytes == 4 << 20
        recv = torch.empty_like(ref_recv)
        rc = lib.ep_dispatch(ctypes.byref(s), ctypes.c_void_p(x.data_ptr()), 0, None, cfg["H"], 0, 0,
                             int(cfg["zero_pad"]), ctypes.c_void_p(recv.data_ptr()), None, stream)
        assert rc == 0
        flags = ctypes.c_uint32(0)
        assert lib.ep_get_status(ctypes.byref(s), stream, ctypes.byref(flags)) == 0 and flags.value == 0

        Np = ref.num_recv_rows()
        assert torch.equal(arrs["cnt"], ref.num_recv_tokens_per_expert)
        assert torch.equal(arrs["off"], ref.expert_offset)
        assert torch.equal(arrs["pair_slot"], ref.pair_slot.view(-1))
        assert torch.equal(arrs["recv_src"][:Np], ref.recv_src_token[:Np])
        assert torch.equal(arrs["recv_w"][:Np].view(torch.int32), ref.recv_weight[:Np].view(torch.int32))
        assert torch.equal(arrs["recv_lexp"][:Np], ref.recv_local_expert[:Np])
        assert np.array_equal(bf16_bits(recv[:Np]), bf16_bits(ref_recv[:Np]))


def test_no_alloc_rejects_sizes_beyond_the_array(ep):
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    cfg = dict(T=256, K=8, E=4096, A=8)              # workspace > 4 MiB
    assert lib.ep_workspace_bytes(256, 8, 4096, 8) > 4 << 20
    s, _ = _handle(cfg, DEV)
    idx = torch.zeros((256, 8), dtype=torch.int64, device=DEV)
    rc = lib.ep_layout_no_alloc(ctypes.c_void_p(idx.data_ptr()), None, 256, 8, 4096, 1, 8, 0, ctypes.byref(s),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ep.EP_ERR_UNSUPPORTED


def _no_alloc(lib, idx, w, T, cfg, s):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ep_layout_no_alloc(ctypes.c_void_p(idx.data_ptr()) if idx is not None else None,
                                  ctypes.c_void_p(w.data_ptr()) if w is not None else None,
                                  T, cfg["K"], cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"],
                                  ctypes.byref(s), stream)


def _dispatch(lib, s, x, H, zero_pad, recv):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ep_dispatch(ctypes.byref(s), ctypes.c_void_p(x.data_ptr()), 0, None, H, 0, 0, int(zero_pad),
                           ctypes.c_void_p(recv.data_ptr()), None, stream)


def test_no_alloc_rejected_call_leaves_the_array_alone(ep):
    """A call that fails its argument checks (T % R != 0) must enqueue nothing:
    the status word and the padding list of the previous call survive it."""
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cfg = workload.config("prefill_bf16")
    inp = workload.inputs(cfg)
    idx, w, x = to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]), to_dev_bf16(inp["x"])
    ref = ep.layout(idx, w, cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"])
    ref_recv = ep.dispatch(ref, x, do_zero_padding=True)
    Np = ref.num_recv_rows()
    assert Np > int((inp["topk_idx"] >= 0).sum())        # the workload has padding rows

    s, _ = _handle(cfg, DEV)
    assert _no_alloc(lib, idx, w, cfg["T"], cfg, s) == 0
    # plant a flag in the shared status word: a bounded wait that runs out
    assert lib.ep_selftest_bounded_wait(ctypes.byref(s), 1_000_000, stream) == 0
    s_bad, _ = _handle(cfg, DEV)
    assert _no_alloc(lib, idx, w, cfg["T"] - 1, cfg, s_bad) == ep.EP_ERR_INVALID_ARG
    assert not s_bad.workspace                            # the rejected handle is unchanged
    flags = ctypes.c_uint32(0)
    assert lib.ep_get_status(ctypes.byref(s), stream, ctypes.byref(flags)) == ep.EP_ERR_TIMEOUT
    assert flags.value == 0x4                             # EP_DEV_TIMEOUT alone
    # the padding list and its length survived too: a zero-padded dispatch
    # into a buffer of 0xff bytes matches ep_layout's, padding rows included
    recv = torch.full_like(ref_recv.view(torch.int16), -1).view(torch.bfloat16)
    assert _dispatch(lib, s, x, cfg["H"], True, recv) == 0
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(recv[:Np]), bf16_bits(ref_recv[:Np]))


def test_no_alloc_zero_tokens(ep):
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cfg = dict(workload.config("prefill_bf16"), T=0)
    s, arrs = _handle(cfg, DEV)
    arrs["cnt"].fill_(7)
    arrs["off"].fill_(7)
    assert _no_alloc(lib, None, None, 0, cfg, s) == 0
    flags = ctypes.c_uint32(1)
    assert lib.ep_get_status(ctypes.byref(s), stream, ctypes.byref(flags)) == 0 and flags.value == 0
    assert int(arrs["cnt"].abs().sum()) == 0 and int(arrs["off"].abs().sum()) == 0
    assert s.num_tokens == 0


def test_no_alloc_older_handle_after_a_newer_call(ep):
    """After a newer no-alloc call, an older no-alloc handle still serves an
    unpadded dispatch and combine: those read only the caller's arrays."""
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cfg1, cfg2 = workload.config("prefill_bf16"), workload.config("decode")
    inp1, inp2 = workload.inputs(cfg1), workload.inputs(cfg2)
    idx1, w1, x1 = to_dev(inp1["topk_idx"]), to_dev(inp1["topk_weights"]), to_dev_bf16(inp1["x"])
    idx2, w2 = to_dev(inp2["topk_idx"]), to_dev(inp2["topk_weights"])
    ref = ep.layout(idx1, w1, cfg1["E"], cfg1["R"], cfg1["A"], cfg1["max_tokens_per_rank"])
    ref_recv = ep.dispatch(ref, x1, do_zero_padding=False)
    ref_out = ep.combine(ref, ref_recv, w1)
    Np = ref.num_recv_rows()
    real = (ref.recv_src_token[:Np] >= 0).cpu().numpy()

    s1, arrs1 = _handle(cfg1, DEV)
    assert _no_alloc(lib, idx1, w1, cfg1["T"], cfg1, s1) == 0
    s2, _ = _handle(cfg2, DEV)
    assert _no_alloc(lib, idx2, w2, cfg2["T"], cfg2, s2) == 0      # replaces the shared array's contents
    recv = torch.zeros_like(ref_recv)
    assert _dispatch(lib, s1, x1, cfg1["H"], False, recv) == 0
    out = torch.empty_like(ref_out)
    rc = lib.ep_combine(ctypes.byref(s1), ctypes.c_void_p(recv.data_ptr()), cfg1["H"],
                        ctypes.c_void_p(w1.data_ptr()), None, None, ctypes.c_void_p(out.data_ptr()), stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(arrs1["pair_slot"], ref.pair_slot.view(-1))
    assert np.array_equal(bf16_bits(recv[:Np])[real], bf16_bits(ref_recv[:Np])[real])
    assert np.array_equal(bf16_bits(out), bf16_bits(ref_out))
