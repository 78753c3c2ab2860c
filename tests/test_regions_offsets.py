"""ep_source_offsets, the host side of expert parallelism over several source
groups (GPUs), checked on the CPU against the oracle's layout of the
concatenated batch (group 0's tokens, then group 1's, ...).

Each group lays out its own tokens with alignment 1 (the oracle stands in for
the group's ep_layout here: the two are bit-identical on the GPU); the groups'
per-expert counts are exchanged - by a real all-gather over world-size-2
`gloo` processes in the second test - and each group's pair (t, k) with expert
e must then land at region e // (E/R), row pair_slot[t, k] + row_delta[e],
which is where the concatenated layout puts it, relative to the region's
first row.  Region sizes and the padding rows are checked the same way.
"""
import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from combine_ep_layout_11_b200 import build, _lib
    build.build()
    return _lib.load()


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def source_offsets(lib, counts, R, A, g):
    """ctypes call of ep_source_offsets; returns (row_delta, region_rows, pad_list)."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    G, E = counts.shape
    delta = np.zeros(E, np.int32)
    rows = np.zeros(R, np.int64)
    npad = ctypes.c_int64(0)
    rc = lib.ep_source_offsets(_ptr(counts), G, E, R, A, g, _ptr(delta), _ptr(rows), None, 0, ctypes.byref(npad))
    assert rc == 0, rc
    pads = np.zeros(max(npad.value, 1), np.int64)
    rc = lib.ep_source_offsets(_ptr(counts), G, E, R, A, g, _ptr(delta), _ptr(rows), _ptr(pads), npad.value,
                               ctypes.byref(npad))
    assert rc == 0, rc
    return delta, rows, pads[:npad.value]


def check_group(idx_g, delta, rows, pads, ref, t0, E, R):
    """Group g's pairs (tokens t0 .. t0 + T_g of the batch) against the concatenated layout."""
    import oracle
    El = E // R
    loc = oracle.layout(idx_g, None, E, R, 1)
    off = ref["off"].astype(np.int64)
    for t in range(idx_g.shape[0]):
        for k in range(idx_g.shape[1]):
            e = int(idx_g[t, k])
            if e < 0:
                assert loc["pair_slot"][t, k] == -1
                continue
            r = e // El
            got = int(loc["pair_slot"][t, k]) + int(delta[e])
            want = int(ref["pair_slot"][t0 + t, k]) - int(off[r * El])
            assert got == want, (t, k, e, got, want)
    assert np.array_equal(rows, off[El::El] - off[:-1:El])
    # padding rows: the rows of each region that hold no pair, as the concatenated layout says
    want = []
    for r in range(R):
        lo, hi = int(off[r * El]), int(off[(r + 1) * El])
        want += [(r << 32) | (row - lo) for row in range(lo, hi) if ref["recv_src"][row] == -1]
    assert np.array_equal(pads, np.array(want, np.int64).reshape(-1))


@pytest.mark.parametrize("G,A,drop", [(2, 128, 0.0), (3, 4, 0.1), (4, 1, 0.3), (1, 16, 0.0)])
def test_offsets_match_the_concatenated_layout(lib, G, A, drop):
    import oracle
    rng = np.random.default_rng(100 + G * 10 + A)
    T_g, K, E, R = 96, 4, 32, 8
    idx = np.stack([rng.permutation(E)[:K] for _ in range(G * T_g)]).astype(np.int64)
    hot = rng.random(idx.shape) < 0.25
    idx[hot] = rng.integers(0, 3, size=int(hot.sum()))      # skew, and repeats inside a token
    idx[rng.random(idx.shape) < drop] = -1
    ref = oracle.layout(idx, None, E, R, A)
    counts = np.stack([oracle.layout(idx[g * T_g:(g + 1) * T_g], None, E, R, 1)["cnt"] for g in range(G)])
    for g in range(G):
        delta, rows, pads = source_offsets(lib, counts, R, A, g)
        check_group(idx[g * T_g:(g + 1) * T_g], delta, rows, pads, ref, g * T_g, E, R)


def test_offsets_argument_checks(lib):
    counts = np.ones((2, 8), np.int32)
    delta = np.zeros(8, np.int32)
    n = ctypes.c_int64(0)
    assert lib.ep_source_offsets(_ptr(counts), 2, 8, 3, 1, 0, _ptr(delta), None, None, 0, None) == 1   # E % R
    assert lib.ep_source_offsets(_ptr(counts), 2, 8, 2, 1, 2, _ptr(delta), None, None, 0, None) == 1   # group
    assert lib.ep_source_offsets(None, 2, 8, 2, 1, 0, _ptr(delta), None, None, 0, None) == 1
    bad = counts.copy()
    bad[1, 3] = -1
    assert lib.ep_source_offsets(_ptr(bad), 2, 8, 2, 1, 0, _ptr(delta), None, None, 0, None) == 1
    small = np.zeros(1, np.int64)
    # 8 experts with 2 pairs each, aligned to 4: 2 padding rows per expert, 16 in all
    assert lib.ep_source_offsets(_ptr(counts), 2, 8, 2, 4, 0, _ptr(delta), None, _ptr(small), 1,
                                 ctypes.byref(n)) == 2
    assert n.value == 16


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    import workload
    from combine_ep_layout_11_b200 import _lib
    lib = _lib.load()
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = workload.config("prefill_bf16")           # 4096 tokens, 256 experts, top-8, R = 8, A = 128
        inp = workload.inputs(cfg)
        E, R, A = cfg["E"], cfg["R"], cfg["A"]
        T_g = cfg["T"] // world
        mine = inp["topk_idx"][rank * T_g:(rank + 1) * T_g]
        local = oracle.layout(mine, None, E, R, 1)
        # the count exchange a multi-GPU dispatch starts with
        gathered = [torch.zeros(E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(local["cnt"].astype(np.int32)))
        counts = torch.stack(gathered).numpy()
        delta, rows, pads = source_offsets(lib, counts, R, A, rank)
        ref = oracle.layout(inp["topk_idx"], None, E, R, A)
        check_group(mine, delta, rows, pads, ref, rank * T_g, E, R)
        dist.barrier()
        out.put((rank, int(rows.sum()), len(pads)))
    finally:
        dist.destroy_process_group()


@pytest.mark.slow
def test_offsets_after_a_gloo_count_all_gather():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    mp.start_processes(_gloo_worker, args=(2, port, q), nprocs=2, join=True, start_method="spawn")
    got = sorted(q.get(timeout=60) for _ in range(2))
    assert got[0][1:] == got[1][1:]                      # both ranks see the same regions
