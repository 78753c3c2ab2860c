"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function raises ``AssertionError`` when the oracle disagrees with
what the pages or the mathematics fix.  The test files call them one by one; the
mutation test re-runs all of them against builds of the oracle with planted
mistakes and requires every mistake to trip at least one pin.

What pins what:
* layout (counts, aligned offsets, slots, inverse maps): exhaustive and random
  brute force against a comparison-sort formulation; the invariants the pages
  fix; the routing-table page's worked examples through the per-rank partition.
* dispatch rows: numpy fancy indexing.
* E4M3 codec: the full 256-code table and torch's float8_e4m3fn conversion
  (a library routine), a hand-derived block, saturation from the definition.
* FP8 cast: torch's float8 conversion of the same formula, the round-trip error
  bound of a 3-bit mantissa, max |q| = 448 per block.
* combine: the fp64-exact sum within the binary32 error bound, identity experts,
  a permutation, hand-derived order / skip examples.
* bf16 rounding: torch's bfloat16 conversion (a library routine).
"""
import functools
import itertools
import json
import os

import numpy as np
import torch

import oracle
import workload

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# layout
# --------------------------------------------------------------------------

def layout_by_sorting(topk_idx, weights, E, R, A):
    """Second formulation of the expand layout: a comparison sort of the pairs by
    (expert, token, k), then each expert's block padded to a multiple of A."""
    T, K = topk_idx.shape
    pairs = sorted((int(topk_idx[t, k]), t, k) for t in range(T) for k in range(K)
                   if topk_idx[t, k] >= 0)
    El = E // R
    rows = []          # (src, weight, lexp) per receive row; None for padding
    slot = {}
    cnt = [0] * E
    off = [0] * (E + 1)
    i = 0
    for e in range(E):
        off[e] = len(rows)
        while i < len(pairs) and pairs[i][0] == e:
            _, t, k = pairs[i]
            slot[(t, k)] = len(rows)
            rows.append((t, 1.0 if weights is None else float(weights[t, k]), e % El))
            cnt[e] += 1
            i += 1
        while (len(rows) - off[e]) % A:
            rows.append(None)
    off[E] = len(rows)
    return cnt, off, slot, rows


def _compare_layout(idx, w, E, R, A):
    lay = oracle.layout(idx, w, E, R, A)
    cnt, off, slot, rows = layout_by_sorting(idx, w, E, R, A)
    assert list(lay["cnt"]) == cnt, (idx.tolist(), E, R, A)
    assert list(lay["off"]) == off, (idx.tolist(), E, R, A)
    T, K = idx.shape
    for t in range(T):
        for k in range(K):
            assert lay["pair_slot"][t, k] == slot.get((t, k), -1), (idx.tolist(), t, k)
    for r, row in enumerate(rows):
        if row is None:
            assert (lay["recv_src"][r], lay["recv_w"][r], lay["recv_lexp"][r]) == (-1, 0.0, -1)
        else:
            assert lay["recv_src"][r] == row[0]
            assert lay["recv_w"][r] == np.float32(row[1])
            assert lay["recv_lexp"][r] == row[2]


def pin_layout_exhaustive():
    """Every topk_idx with T*K <= 4 entries in {-1, 0..E-1}, E in {2, 4}."""
    for E in (2, 4):
        for (T, K) in [(1, 1), (1, 2), (2, 1), (2, 2), (1, 4), (4, 1), (1, 3), (3, 1)]:
            for R in (1, 2):
                if E % R or T % R:
                    continue
                for A in (1, 2, 3):
                    for vals in itertools.product(range(-1, E), repeat=T * K):
                        idx = np.array(vals, np.int64).reshape(T, K)
                        _compare_layout(idx, None, E, R, A)


def pin_layout_random(n=300, seed=7):
    rng = np.random.default_rng(seed)
    for _ in range(n):
        R = int(rng.choice([1, 2, 4]))
        E = R * int(rng.integers(1, 5))
        T = R * int(rng.integers(0, 6))
        K = int(rng.integers(1, 5))
        A = int(rng.integers(1, 6))
        idx = rng.integers(-1, E, (T, K)).astype(np.int64)
        w = rng.random((T, K)).astype(np.float32)
        _compare_layout(idx, w, E, R, A)


def check_layout_invariants(lay, topk_idx, topk_weights, E, R, A):
    """The invariants the pages fix, on any size."""
    T, K = topk_idx.shape
    sel = topk_idx >= 0
    N = int(sel.sum())
    cnt, off, ps = lay["cnt"], lay["off"], lay["pair_slot"]
    # pairs = T*K minus the -1 entries; counts sum to the receive size before padding
    assert N == T * K - int((topk_idx == -1).sum())
    assert int(cnt.sum()) == N
    assert np.array_equal(cnt, np.bincount(topk_idx[sel], minlength=E))
    # every aligned offset is a multiple of expert_alignment
    assert np.all(off % A == 0)
    assert np.array_equal(np.diff(off), (cnt + A - 1) // A * A)
    Np = int(off[E])
    # slots are injective; with the padding rows they tile [0, Np)
    slots = ps[sel]
    assert np.all(ps[~sel] == -1)
    assert np.unique(slots).size == N and (N == 0 or (slots.min() >= 0 and slots.max() < Np))
    pad = lay["recv_src"][:Np] == -1
    assert int(pad.sum()) == Np - N
    covered = np.zeros(Np, bool)
    covered[slots] = True
    assert np.array_equal(covered, ~pad)
    # inverse maps
    tt = np.repeat(np.arange(T), K).reshape(T, K)
    assert np.array_equal(lay["recv_src"][slots], tt[sel])
    assert np.array_equal(lay["recv_lexp"][slots], topk_idx[sel] % (E // R))
    if topk_weights is not None:
        assert np.array_equal(lay["recv_w"][slots], topk_weights[sel])
    assert np.all(lay["recv_lexp"][:Np][pad] == -1) and np.all(lay["recv_w"][:Np][pad] == 0)
    # each expert's rows lie in [off[e], off[e+1]) and hold its pairs in token order
    e_of_pair = topk_idx[sel]
    assert np.all(slots >= off[e_of_pair]) and np.all(slots < off[e_of_pair] + cnt[e_of_pair])
    for e in np.nonzero(cnt > 1)[0][:64]:
        src = lay["recv_src"][off[e]:off[e] + cnt[e]]
        assert np.all(np.diff(src) >= 0)
    # per source rank: local + remote = that rank's pairs; the receive region of
    # rank r holds exactly the pairs whose expert r owns (routing-table page)
    El, Tr = E // R, T // R
    tot_local = tot_remote = 0
    for r in range(R):
        tab = oracle.routing_table(topk_idx[r * Tr:(r + 1) * Tr],
                                   np.zeros((Tr, K), np.float32) if topk_weights is None
                                   else topk_weights[r * Tr:(r + 1) * Tr],
                                   Tr, K, r * El, (r + 1) * El)
        n_r = int(sel[r * Tr:(r + 1) * Tr].sum())
        nl, nr = len(tab["local_token_indices"]), len(tab["remote_token_indices"])
        assert nl + nr == n_r
        region = slice(off[r * El], off[(r + 1) * El])
        src = lay["recv_src"][region]
        assert int(((src >= r * Tr) & (src < (r + 1) * Tr)).sum()) == nl
        assert int(cnt[r * El:(r + 1) * El].sum()) == int((src >= 0).sum())
        tot_local += nl
        tot_remote += nr
    assert tot_local + tot_remote == N


@functools.lru_cache(maxsize=None)
def _routing(name):
    return workload.routing(workload.config(name))


def pin_layout_invariants_workloads(names=("tiny", "prefill_bf16", "decode", "large_prefill")):
    for name in names:
        cfg = workload.config(name)
        idx, w = _routing(name)
        lay = oracle.layout(idx, w, cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"])
        check_layout_invariants(lay, idx, w, cfg["E"], cfg["R"], cfg["A"])


def pin_layout_errors():
    idx = np.array([[0, 1], [2, 3]], np.int64)
    for bad in (-2, 4, 1 << 40):
        b = idx.copy()
        b[1, 0] = bad
        try:
            oracle.layout(b, None, 4, 2, 1)
            raise AssertionError("bad expert id %d accepted" % bad)
        except oracle.OracleError as exc:
            assert exc.code == oracle.ERR_BAD_EXPERT
    for args in [(4, 3, 1), (4, 2, 0), (3, 2, 1)]:     # E % R, A < 1, E % R
        try:
            oracle.layout(idx, None, *args)
            raise AssertionError("invalid arguments accepted: %r" % (args,))
        except oracle.OracleError as exc:
            assert exc.code == oracle.ERR_INVALID_ARG
    try:                                               # T / R above the per-rank limit
        oracle.layout(idx, None, 4, 1, 1, num_max_tokens_per_rank=1)
        raise AssertionError("per-rank token limit not enforced")
    except oracle.OracleError as exc:
        assert exc.code == oracle.ERR_CAPACITY
    try:                                               # receive rows above capacity
        oracle.layout(idx, None, 4, 2, 2, capacity=7)
        raise AssertionError("capacity not enforced")
    except oracle.OracleError as exc:
        assert exc.code == oracle.ERR_CAPACITY
    lay = oracle.layout(idx, None, 4, 2, 2, capacity=8)
    assert int(lay["off"][-1]) == 8


def pin_routing_table_golden():
    g = _golden("routing_table_examples.json")
    for case in g["cases"]:
        exp = case["expect"]
        try:
            tab = oracle.routing_table(case["indices"], case["weights"], case["num_tokens"],
                                       case["top_k"], case["local_start"], case["local_end"])
        except oracle.OracleError as exc:
            assert exp.get("error") == exc.code, (case["name"], exc.code)
            continue
        assert "error" not in exp, case["name"]
        nl, nr = len(tab["local_token_indices"]), len(tab["remote_token_indices"])
        assert exp.get("local_count", nl) == nl, case["name"]
        assert exp.get("remote_count", nr) == nr, case["name"]
        assert exp.get("total_count", nl + nr) == nl + nr, case["name"]
        for key in ("local_token_indices", "local_expert_ids", "remote_token_indices",
                    "remote_expert_ids"):
            if key in exp:
                assert tab[key].tolist() == exp[key], (case["name"], key)
        for key in ("local_weights", "remote_weights"):
            if key in exp:
                assert np.array_equal(tab[key], np.array(exp[key], np.float32)), (case["name"], key)


# --------------------------------------------------------------------------
# dispatch rows
# --------------------------------------------------------------------------

def pin_dispatch_rows(seed=11):
    rng = np.random.default_rng(seed)
    for (T, K, E, R, A, zp) in [(8, 2, 4, 2, 3, True), (16, 4, 8, 4, 4, False), (6, 3, 6, 3, 2, True),
                                (0, 2, 4, 2, 2, True)]:
        idx = rng.integers(-1, E, (T, K)).astype(np.int64)
        x = rng.integers(0, 1 << 16, (T, 24), dtype=np.uint16)
        lay = oracle.layout(idx, None, E, R, A)
        recv = oracle.dispatch_rows(x, lay, zp, fill=0xA5)
        expect = np.full((lay["capacity"], 24), 0xA5A5, np.uint16)
        sel = idx >= 0
        tt = np.repeat(np.arange(T), K).reshape(T, K)
        expect[lay["pair_slot"][sel]] = x[tt[sel]]
        if zp:
            Np = int(lay["off"][-1])
            pad = np.nonzero(lay["recv_src"][:Np] == -1)[0]
            expect[pad] = 0
        assert np.array_equal(recv, expect)


# --------------------------------------------------------------------------
# E4M3 codec and the FP8 cast
# --------------------------------------------------------------------------

def _torch_e4m3(v):
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def pin_e4m3_decode_table():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def e4m3_test_values(seed=3):
    """All finite bf16 values below the non-saturating limit, every E4M3 midpoint
    and its binary32 neighbours, and random binary32 values."""
    allbf = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    allbf = allbf[np.isfinite(allbf) & (np.abs(allbf) < 464.0)]
    mags = np.sort(oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64))
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)
    nb = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    rng = np.random.default_rng(seed)
    rnd = (rng.standard_normal(200000) * np.exp2(rng.integers(-12, 9, 200000))).astype(np.float32)
    rnd = rnd[np.abs(rnd) < 464.0]
    v = np.concatenate([allbf, nb, -nb, rnd])
    return v


def pin_e4m3_encode_vs_torch():
    v = e4m3_test_values()
    assert np.array_equal(oracle.e4m3_encode(v), _torch_e4m3(v))


def pin_e4m3_saturation():
    big = np.array([448.0, 460.0, 464.0, 479.9, 480.0, 1e4, 3.0e38, np.inf], np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    assert (int(oracle.e4m3_encode(np.array([np.nan], np.float32))[0]) & 0x7F) == 0x7F


def pin_fp8_golden_block():
    g = _golden("fp8_block_example.json")
    H = g["H"]
    x = np.zeros((1, H), np.float32)
    x[0, :len(g["block0_values"])] = g["block0_values"]
    xb = workload.to_bf16_bits(x)
    assert np.array_equal(oracle.bf16_to_f32(xb), x), "golden values must be bf16-exact"
    q, s = oracle.cast_fp8(xb)
    n = len(g["block0_codes"])
    assert q[0, :n].tolist() == g["block0_codes"]
    assert np.all(q[0, n:128] == 0) and np.all(q[0, 128:] == 0)
    assert s[0, 0] == np.float32(g["block0_scale"])
    assert s[0, 1] == np.float32(1e-4) / np.float32(448.0)


def _torch_cast(xb):
    """The pages' formula through torch (binary32 division, torch's float8 conversion)."""
    T, H = xb.shape
    xf = torch.from_numpy(oracle.bf16_to_f32(xb).reshape(T, H // 128, 128))
    amax = xf.abs().amax(dim=2).clamp_min(1e-4)
    s = amax / 448.0
    q = (xf / s.unsqueeze(2)).to(torch.float8_e4m3fn).view(torch.uint8)
    return q.reshape(T, H).numpy(), s.numpy()


def cast_test_inputs(seed=5):
    rng = np.random.default_rng(seed)
    x1 = workload.to_bf16_bits(rng.standard_normal((64, 1024), dtype=np.float32))
    x2 = workload.to_bf16_bits((rng.standard_normal((64, 1024)) *
                                np.exp2(rng.integers(-30, 30, (64, 1024)))).astype(np.float32))
    # every bf16 magnitude in [2^-20, 2) under a fixed block maximum 2.0
    allbf = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    pool = allbf[np.isfinite(allbf) & (np.abs(allbf) < 2.0) & (np.abs(allbf) > 2.0 ** -20)]
    pool = pool[: (pool.size // 127) * 127].reshape(-1, 127)
    blocks = np.concatenate([np.full((pool.shape[0], 1), 2.0, np.float32), pool], axis=1)
    blocks = blocks[: (blocks.shape[0] // 8) * 8].reshape(-1, 1024)
    x3 = workload.to_bf16_bits(blocks)
    # a few all-zero and tiny blocks (amax clamp)
    x4 = np.zeros((2, 1024), np.uint16)
    x4[1, :128] = workload.to_bf16_bits(np.full(128, 1e-6, np.float32))
    return np.concatenate([x1, x2, x3, x4])


def pin_cast_vs_torch():
    xb = cast_test_inputs()
    q, s = oracle.cast_fp8(xb)
    tq, ts = _torch_cast(xb)
    assert np.array_equal(s.view(np.uint32), ts.view(np.uint32))
    assert np.array_equal(q, tq)


def pin_cast_roundtrip():
    xb = cast_test_inputs()
    T, H = xb.shape
    q, s = oracle.cast_fp8(xb)
    x = oracle.bf16_to_f32(xb).astype(np.float64)
    d = oracle.dequant_fp8(q, s).astype(np.float64)
    sb = np.repeat(s.astype(np.float64), 128, axis=1)
    # 3 mantissa bits: half-spacing <= 2^-4 |v| for normals, 2^-10 in the subnormal range
    bound = np.maximum(np.abs(x) * 2.0 ** -4, sb * 2.0 ** -10) * (1 + 2.0 ** -18) + sb * 2.0 ** -30
    assert np.all(np.abs(d - x) <= bound)
    # the block maximum maps to +-448 unless the block is below the amax clamp
    qb = np.abs(oracle.e4m3_decode(q)).reshape(T, H // 128, 128).max(axis=2)
    amax = np.abs(x).reshape(T, H // 128, 128).max(axis=2)
    assert np.all(qb[amax >= 1e-4] == 448.0)


def _torch_cast_variant(xb, per_row, round_scale):
    """The pages' formula through torch, with the group width and the
    power-of-two rounding of the scale written with torch's log2 / ceil / exp2."""
    T, H = xb.shape
    g = H if per_row else 128
    xf = torch.from_numpy(oracle.bf16_to_f32(xb).reshape(T, H // g, g))
    amax = xf.abs().amax(dim=2).clamp_min(1e-4)
    s = amax / 448.0
    if round_scale:
        s = torch.exp2(torch.ceil(torch.log2(s.double()))).float()
    q = (xf / s.unsqueeze(2)).to(torch.float8_e4m3fn).view(torch.uint8)
    return q.reshape(T, H).numpy(), s.numpy()


def _variant_inputs():
    xb = cast_test_inputs()
    # blocks whose amax / 448 is exactly a power of two (amax = 1.75 * 2^j)
    rng = np.random.default_rng(29)
    x5 = (rng.uniform(-1, 1, (16, 1024)) * 1.75).astype(np.float32)
    x5[:, ::128] = np.float32(1.75) * np.exp2(rng.integers(-20, 20, (16, 8))).astype(np.float32)
    return np.concatenate([xb, workload.to_bf16_bits(x5)])


def pin_cast_variants_vs_torch():
    xb = _variant_inputs()
    for per_row in (False, True):
        for round_scale in (False, True):
            q, s = oracle.cast_fp8(xb, per_row=per_row, round_scale=round_scale)
            tq, ts = _torch_cast_variant(xb, per_row, round_scale)
            assert np.array_equal(s.view(np.uint32), ts.view(np.uint32)), (per_row, round_scale)
            assert np.array_equal(q, tq), (per_row, round_scale)


def pin_round_scale_properties():
    """A rounded scale is a power of two, not below amax / 448 and below twice it."""
    xb = _variant_inputs()
    for per_row in (False, True):
        _, s0 = oracle.cast_fp8(xb, per_row=per_row)
        _, s1 = oracle.cast_fp8(xb, per_row=per_row, round_scale=True)
        m, _ = np.frexp(s1.astype(np.float64))
        assert np.all(m == 0.5)
        assert np.all(s1 >= s0) and np.all(s1.astype(np.float64) / 2 < s0)


def pin_fp8_variants_golden():
    g = _golden("fp8_variants_example.json")
    x = np.zeros((1, g["H"]), np.float32)
    x[0, :len(g["block0_values"])] = g["block0_values"]
    x[0, 128:128 + len(g["block1_values"])] = g["block1_values"]
    xb = workload.to_bf16_bits(x)
    assert np.array_equal(oracle.bf16_to_f32(xb), x), "golden values must be bf16-exact"
    n0, n1 = len(g["block0_values"]), len(g["block1_values"])
    q, s = oracle.cast_fp8(xb, round_scale=True)
    assert q[0, :n0].tolist() == g["block_round"]["block0_codes"]
    assert q[0, 128:128 + n1].tolist() == g["block_round"]["block1_codes"]
    assert s[0].tolist() == g["block_round"]["scales"]
    assert oracle.ue8m0_encode(s)[0].tolist() == g["block_round"]["ue8m0"]
    q, s = oracle.cast_fp8(xb, per_row=True, round_scale=True)
    assert s.shape == (1, 1) and float(s[0, 0]) == g["row_round"]["scale"]
    assert q[0, :n0].tolist() == g["block_round"]["block0_codes"]
    assert q[0, 128:128 + n1].tolist() == g["row_round"]["block1_codes"]
    assert int(oracle.ue8m0_encode(s)[0, 0]) == g["row_round"]["ue8m0"]


def pin_ue8m0():
    b = np.arange(255, dtype=np.uint8)
    v = oracle.ue8m0_decode(b)
    assert np.array_equal(v.astype(np.float64), np.exp2(b.astype(np.float64) - 127))
    assert np.array_equal(oracle.ue8m0_encode(v), b)
    for bad in (3.0, 0.75, 1.5 * 2.0 ** -20):
        try:
            oracle.ue8m0_encode(np.array([bad], np.float32))
        except oracle.OracleError:
            continue
        raise AssertionError("UE8M0 accepted a scale that is not a power of two: %r" % bad)


def pin_cast_variants_roundtrip():
    xb = _variant_inputs()
    T, H = xb.shape
    x = oracle.bf16_to_f32(xb).astype(np.float64)
    for per_row in (False, True):
        for round_scale in (False, True):
            q, s = oracle.cast_fp8(xb, per_row=per_row, round_scale=round_scale)
            d = oracle.dequant_fp8(q, s).astype(np.float64)
            sb = np.repeat(s.astype(np.float64), H // s.shape[1], axis=1)
            bound = np.maximum(np.abs(x) * 2.0 ** -4, sb * 2.0 ** -10) * (1 + 2.0 ** -18) + sb * 2.0 ** -30
            assert np.all(np.abs(d - x) <= bound), (per_row, round_scale)
            assert np.all(np.abs(oracle.e4m3_decode(q)) <= 448.0)


def pin_scales_col_major():
    rng = np.random.default_rng(31)
    for rows, G, dt in [(1, 1, np.float32), (5, 3, np.float32), (8, 56, np.float32), (17, 2, np.uint8),
                        (32, 7, np.uint8)]:
        sc = rng.integers(1, 200, (rows, G)).astype(dt)
        cm = oracle.scales_col_major(sc)
        per16 = 16 // np.dtype(dt).itemsize
        assert cm.shape[0] == G and cm.shape[1] % per16 == 0 and rows <= cm.shape[1] < rows + per16
        flat = cm.reshape(-1)
        for r in range(rows):
            for g in range(G):
                assert flat[g * cm.shape[1] + r] == sc[r, g]


def pin_bf16_rounding():
    rng = np.random.default_rng(9)
    u = rng.integers(0, 1 << 32, 400000, dtype=np.uint64).astype(np.uint32)
    ties = ((rng.integers(0, 1 << 16, 2000, dtype=np.uint32) << 16) | 0x8000).astype(np.uint32)
    v = np.concatenate([u, ties]).view(np.float32)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(v), ref)


# --------------------------------------------------------------------------
# combine
# --------------------------------------------------------------------------

def pin_combine_golden():
    g = _golden("combine_examples.json")
    for case in g["cases"]:
        y = np.array(case["y_bits"], np.uint16)
        ps = np.array(case["pair_slot"], np.int32)
        w = None if case["weights"] is None else np.array(case["weights"], np.float32)
        b0 = np.array(case["bias0_bits"], np.uint16) if "bias0_bits" in case else None
        b1 = np.array(case["bias1_bits"], np.uint16) if "bias1_bits" in case else None
        out = oracle.combine(y, ps, w, b0, b1)
        assert out.tolist() == case["out_bits"], case["name"]


def _rand_bf16(rng, shape, lo=-60, hi=60):
    """Random signs and mantissas, exponents in [lo, hi]: no overflow, no subnormals."""
    return ((rng.integers(0, 2, shape, dtype=np.uint16) << 15)
            | (rng.integers(127 + lo, 127 + hi + 1, shape, dtype=np.uint16) << 7)
            | rng.integers(0, 128, shape, dtype=np.uint16)).astype(np.uint16)


def pin_combine_fp64_bound(seed=13):
    rng = np.random.default_rng(seed)
    for (T, K, rows, H, weighted, nbias) in [(64, 8, 300, 64, True, 0), (32, 4, 50, 40, False, 0),
                                             (16, 1, 16, 8, True, 0), (48, 8, 200, 32, True, 1),
                                             (24, 4, 80, 16, False, 2)]:
        # random signs and mantissas, exponents in [-60, 60]: no overflow, no subnormal products
        y = _rand_bf16(rng, (rows, H))
        ps = rng.integers(-1, rows, (T, K)).astype(np.int32)
        w = (rng.standard_normal((T, K)) * 2).astype(np.float32) if weighted else None
        biases = [_rand_bf16(rng, (T, H)) for _ in range(nbias)] + [None] * (2 - nbias)
        out = oracle.combine(y, ps, w, biases[0], biases[1])
        yf = oracle.bf16_to_f32(y).astype(np.float64)
        wf = np.ones((T, K)) if w is None else w.astype(np.float64)
        sel = ps >= 0
        terms = np.where(sel[:, :, None], wf[:, :, None] * yf[np.maximum(ps, 0)], 0.0)
        bsum = sum(oracle.bf16_to_f32(b).astype(np.float64) for b in biases if b is not None)
        exact = terms.sum(axis=1) + bsum
        mag = np.abs(terms).sum(axis=1) + sum(np.abs(oracle.bf16_to_f32(b).astype(np.float64))
                                              for b in biases if b is not None)
        got = oracle.bf16_to_f32(out).astype(np.float64)
        u = 2.0 ** -24
        n = 2 * K + nbias                 # K products, K + nbias - 1 additions, at most
        gamma = n * u / (1 - n * u)
        bound = 2.0 ** -8 * np.abs(exact) * (1 + gamma) + (1 + 2.0 ** -8) * gamma * mag + 1e-40
        assert np.all(np.abs(got - exact) <= bound)


def pin_combine_identity():
    """Identity experts: y = dispatched x; weights renormalised over the selected
    entries sum to 1, so combine reproduces x (0 for all-unselected tokens)."""
    rng = np.random.default_rng(17)
    for (T, H, E, K, R, A) in [(64, 256, 16, 4, 4, 4), (32, 128, 8, 8, 2, 1)]:
        idx = rng.integers(-1, E, (T, K)).astype(np.int64)
        idx[0] = -1
        w = rng.random((T, K)).astype(np.float32) + 0.1
        w = np.where(idx >= 0, w, 0).astype(np.float32)
        s = w.sum(axis=1, keepdims=True)
        w = np.where(s > 0, w / np.where(s > 0, s, 1), 0).astype(np.float32)
        x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
        lay = oracle.layout(idx, w, E, R, A)
        y = oracle.dispatch_rows(x, lay, True)
        out = oracle.combine(y, lay["pair_slot"], w)
        has = (idx >= 0).any(axis=1)
        assert np.array_equal(out[has], x[has])
        assert np.all(out[~has] == 0)


def pin_combine_permutation():
    rng = np.random.default_rng(19)
    T, H, rows = 40, 32, 60
    y = rng.integers(0, 1 << 16, (rows, H), dtype=np.uint16)
    y[(y & 0x7F80) == 0x7F80] = 0x3F80
    y[(y & 0x7FFF) == 0] = 0x3F80                    # -0 would turn into +0 via 0 + (-0)
    ps = rng.permutation(rows)[:T].astype(np.int32).reshape(T, 1)
    assert np.array_equal(oracle.combine(y, ps, None), y[ps[:, 0]])


def pin_recv_stats():
    """cumulative_local_expert_recv_stats over two calls = the two histograms summed."""
    rng = np.random.default_rng(23)
    E = 16
    stats = rng.integers(0, 100, E).astype(np.int32)
    start = stats.copy()
    seen = np.zeros(E, np.int64)
    for _ in range(2):
        idx = rng.integers(-1, E, (40, 4)).astype(np.int64)
        lay = oracle.layout(idx, None, E, 4, 8)
        stats = oracle.accumulate_recv_stats(stats, lay["cnt"])
        seen += np.bincount(idx[idx >= 0], minlength=E)
    assert np.array_equal(stats, start + seen)


def _rank_layout_numpy(idx, w, E, R, A):
    """The per-token-per-rank layout restated with numpy set operations."""
    T, K = idx.shape
    El = E // R
    dest = np.where(idx >= 0, idx // El, -1)
    in_rank = (dest[:, :, None] == np.arange(R)[None, None, :]).any(axis=1)
    tokens = [np.nonzero(in_rank[:, r])[0] for r in range(R)]
    n_rank = np.array([len(tk) for tk in tokens], np.int32)
    rank_off = np.concatenate([[0], np.cumsum(n_rank)]).astype(np.int32)
    token_slot = np.full((T, R), -1, np.int32)
    for r in range(R):
        token_slot[tokens[r], r] = rank_off[r] + np.arange(len(tokens[r]))
    src = np.concatenate(tokens + [np.zeros(0, np.int64)]).astype(np.int32)
    row_rank = np.repeat(np.arange(R), n_rank)
    local = dest[src] == row_rank[:, None]
    ridx = np.where(local, idx[src] - row_rank[:, None] * El, -1)
    ww = np.ones((T, K), np.float32) if w is None else w
    rw = np.where(local, ww[src], 0).astype(np.float32)
    n_exp = np.bincount(idx[idx >= 0], minlength=E).astype(np.int32)
    n_recv = ((n_exp + A - 1) // A * A).astype(np.int32)
    return dict(is_token_in_rank=in_rank, num_tokens_per_rank=n_rank, rank_off=rank_off, token_slot=token_slot,
                recv_src=src, recv_topk_idx=ridx, recv_topk_weights=rw, num_tokens_per_expert=n_exp,
                num_recv_tokens_per_expert=n_recv)


def pin_rank_layout_vs_numpy(n=120, seed=37):
    rng = np.random.default_rng(seed)
    for i in range(n):
        R = int(rng.choice([1, 2, 4, 8]))
        E = R * int(rng.integers(1, 5))
        T = R * int(rng.integers(0, 9))
        K = int(rng.integers(1, 6))
        A = int(rng.integers(1, 4))
        idx = rng.integers(-1, E, (T, K)).astype(np.int64)
        w = rng.random((T, K)).astype(np.float32) if i % 2 else None
        got = oracle.rank_layout(idx, w, E, R, A)
        exp = _rank_layout_numpy(idx, w, E, R, A)
        rows = int(exp["rank_off"][-1])
        for key in ("is_token_in_rank", "num_tokens_per_rank", "rank_off", "token_slot",
                    "num_tokens_per_expert", "num_recv_tokens_per_expert"):
            assert np.array_equal(got[key], exp[key]), key
        assert np.array_equal(got["recv_src"][:rows], exp["recv_src"])
        assert np.array_equal(got["recv_topk_idx"][:rows], exp["recv_topk_idx"])
        assert np.array_equal(got["recv_topk_weights"][:rows].view(np.uint32),
                              exp["recv_topk_weights"].view(np.uint32))


def pin_rank_layout_exhaustive():
    """Every topk_idx with T*K <= 4 entries in {-1, 0..E-1}, E in {2, 4}, R in {1, 2, 4},
    against the numpy restatement."""
    for E in (2, 4):
        for (T, K) in [(1, 1), (2, 1), (2, 2), (4, 1), (1, 3), (1, 4)]:
            for R in (1, 2, 4):
                if E % R or T % R:
                    continue
                for vals in itertools.product(range(-1, E), repeat=T * K):
                    idx = np.array(vals, np.int64).reshape(T, K)
                    got = oracle.rank_layout(idx, None, E, R, 2)
                    exp = _rank_layout_numpy(idx, None, E, R, 2)
                    rows = int(exp["rank_off"][-1])
                    for key in ("is_token_in_rank", "num_tokens_per_rank", "rank_off", "token_slot",
                                "num_tokens_per_expert", "num_recv_tokens_per_expert"):
                        assert np.array_equal(got[key], exp[key]), (key, idx.tolist(), R)
                    assert np.array_equal(got["recv_src"][:rows], exp["recv_src"])
                    assert np.array_equal(got["recv_topk_idx"][:rows], exp["recv_topk_idx"])


def pin_rank_layout_golden():
    g = _golden("rank_layout_example.json")
    d = oracle.rank_layout(np.array(g["topk_idx"], np.int64), np.array(g["topk_weights"], np.float32),
                           g["E"], g["R"], g["A"])
    rows = sum(g["num_tokens_per_rank"])
    for key in ("num_tokens_per_rank", "token_slot", "num_tokens_per_expert", "num_recv_tokens_per_expert"):
        assert d[key].tolist() == g[key], key
    assert d["is_token_in_rank"].astype(int).tolist() == g["is_token_in_rank"]
    assert d["recv_src"][:rows].tolist() == g["recv_src"]
    assert d["recv_topk_idx"][:rows].tolist() == g["recv_topk_idx"]
    assert d["recv_topk_weights"][:rows].tolist() == g["recv_topk_weights"]


def pin_rank_layout_matches_expand():
    """Same routing, both forms: per-expert counts agree with the expand layout,
    and the local entries of rank r's rows are exactly the pairs the expand
    layout puts in rank r's region."""
    for name in ("tiny", "prefill_bf16"):
        cfg = workload.config(name)
        idx, w = workload.routing(cfg)
        E, R, A = cfg["E"], cfg["R"], cfg["A"]
        ex = oracle.layout(idx, w, E, R, A)
        rk = oracle.rank_layout(idx, w, E, R, A)
        assert np.array_equal(rk["num_tokens_per_expert"], ex["cnt"])
        assert np.array_equal(rk["num_recv_tokens_per_expert"], np.diff(ex["off"]))
        El = E // R
        for r in range(R):
            lo, hi = rk["rank_off"][r], rk["rank_off"][r + 1]
            ri = rk["recv_topk_idx"][lo:hi]
            pairs = int((ri >= 0).sum())
            assert pairs == int(ex["cnt"][r * El:(r + 1) * El].sum())


def pin_rank_combine_identity():
    """Rank-level combine (§3.2: plain sum over the reached ranks, K = R, unit
    weights): expert outputs equal to x on each token's first rank and 0 on
    the others reproduce x."""
    rng = np.random.default_rng(41)
    T, K, E, R, H = 48, 4, 16, 4, 64
    idx = rng.integers(-1, E, (T, K)).astype(np.int64)
    idx[0] = -1
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    rk = oracle.rank_layout(idx, None, E, R, 1)
    y = np.zeros((rk["capacity"], H), np.uint16)
    for t in range(T):
        slots = rk["token_slot"][t][rk["token_slot"][t] >= 0]
        if slots.size:
            y[slots[0]] = x[t]
    out = oracle.combine(y, rk["token_slot"], None)
    has = rk["is_token_in_rank"].any(axis=1)
    expect = np.where(x == 0x8000, np.uint16(0), x)
    assert np.array_equal(out[has], expect[has]) and np.all(out[~has] == 0)


def pin_ll_layout_golden():
    g = _golden("ll_layout_example.json")
    lay = oracle.ll_layout(np.array(g["topk_idx"], np.int64), None, g["E"], g["R"], g["max_tokens"])
    assert lay["cnt"].tolist() == g["cnt"] and lay["off"].tolist() == g["off"]
    assert lay["pair_slot"].tolist() == g["pair_slot"] and lay["recv_src"].tolist() == g["recv_src"]
    # more pairs for one expert than its slab holds: a capacity error
    try:
        oracle.ll_layout(np.zeros((2, 2), np.int64), None, 2, 1, 2)     # 4 pairs, slab of 2
    except oracle.OracleError as err:
        assert err.code == 2
    else:
        raise AssertionError("slab overflow not reported")


def pin_ll_layout_vs_expand(n=80, seed=43):
    """The fixed-slab form is the A = 1 expand layout with every expert moved to
    e * S: same counts, same order within an expert, padding to the slab end."""
    rng = np.random.default_rng(seed)
    for i in range(n):
        R = int(rng.choice([1, 2, 4]))
        E = R * int(rng.integers(1, 5))
        T = R * int(rng.integers(0, 6))
        K = int(rng.integers(1, 4))
        M = max(T // R, 1) + int(rng.integers(0, 3))
        idx = rng.integers(-1, E, (T, K)).astype(np.int64)
        w = rng.random((T, K)).astype(np.float32)
        S = R * M
        ex = oracle.layout(idx, w, E, R, 1)
        try:
            ll = oracle.ll_layout(idx, w, E, R, M)
        except oracle.OracleError as err:
            assert err.code == 2 and (ex["cnt"] > S).any()        # an expert overflows its slab
            continue
        assert np.array_equal(ll["cnt"], ex["cnt"])
        assert np.array_equal(ll["off"], np.arange(E + 1) * S)
        e_of = np.where(idx >= 0, idx, 0)
        sel = idx >= 0
        assert np.array_equal((ll["pair_slot"] - ll["off"][e_of])[sel], (ex["pair_slot"] - ex["off"][e_of])[sel])
        assert np.all(ll["pair_slot"][~sel] == -1)
        for e in range(E):
            pad = ll["recv_src"][e * S + ll["cnt"][e]:(e + 1) * S]
            assert np.all(pad == -1)


ALL_PINS = [
    pin_layout_exhaustive, pin_layout_random, pin_layout_invariants_workloads, pin_layout_errors,
    pin_routing_table_golden, pin_dispatch_rows, pin_e4m3_decode_table, pin_e4m3_encode_vs_torch,
    pin_e4m3_saturation, pin_fp8_golden_block, pin_cast_vs_torch, pin_cast_roundtrip,
    pin_bf16_rounding, pin_combine_golden, pin_combine_fp64_bound, pin_combine_identity,
    pin_combine_permutation, pin_recv_stats,
    pin_cast_variants_vs_torch, pin_round_scale_properties, pin_fp8_variants_golden, pin_ue8m0,
    pin_cast_variants_roundtrip, pin_scales_col_major,
    pin_rank_layout_vs_numpy, pin_rank_layout_exhaustive, pin_rank_layout_golden, pin_rank_layout_matches_expand,
    pin_rank_combine_identity,
    pin_ll_layout_golden, pin_ll_layout_vs_expand,
]
