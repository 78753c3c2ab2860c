"""ep_layout_no_alloc, the layout entry point for callers that cannot allocate
device memory themselves (a plain C host program with no device allocator of
its own, or a process whose device memory belongs to another framework's
pool): its workspace is a fixed array in the library's own device memory.

Through the C ABI, two calls in a row (different workloads, so stale contents
of the shared array would show) must give the same bytes as ep_layout with a
caller-owned workspace, and a dispatch on the returned handle must match too.
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
                pair_slot=torch.empty(T * K, dtype=torch.int32, device=dev),
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
