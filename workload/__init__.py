"""Seeded synthetic inputs for MoE dispatch / combine.

This module is shared by the tests, the benchmark and the oracle's checks.  It
only makes inputs (routing indices, routing weights, token rows, expert outputs)
and holds none of the dispatch / combine arithmetic.

The five workloads follow the shapes of the DeepEP pages: H = 7168 hidden,
256 experts, top-8 routing with skewed gate scores, R virtual ranks that each own
E / R contiguous experts ("DeepEP 测试目标 API 系统性参考", §2.1 dispatch()
parameter table and §4.3 gate.py).  Recipe:

* token rows x ~ N(0, 1), rounded to bf16 (nearest even);
* gate scores: U(0, 1) for the uniform gates, N(0, 1) + b_e for the skewed ones,
  where expert e has popularity rank i = pi(e) + 1 under a seeded permutation pi
  and b_e = beta * (-s * ln i) (a Zipf(s) log-popularity bias);
* beta is found by bisection, as gate.py's ratio search does, so that in the
  large-prefill workload (s = 1.5) the two most loaded experts take 20 % of the
  pairs; the same beta serves the s = 1.2 workloads;
* topk_idx = the K highest scores, best first (ties to the lower expert id);
  topk_weights = softmax over those K scores, in fp64, rounded to fp32;
* the decode workload sets each topk_idx entry to -1 independently with p = 0.1
  (its weight is kept, so a consumer that fails to skip -1 entries is caught);
* expert outputs (the combine input) are seeded random bf16 values with
  exponents in [-7, 3], i.e. magnitudes in [2^-7, 16).

Seeds are 1000 + the workload's position (1..5); independent streams for the
gate, the drop mask, x and y come from ``numpy.random.SeedSequence.spawn``.
"""
import functools

import numpy as np

WORKLOADS = {
    "tiny": dict(index=1, T=128, H=256, E=16, K=4, R=2, A=1, zero_pad=False, fp8=False,
                 gate="uniform", zipf_s=None, drop=0.0, max_tokens_per_rank=0),
    "prefill_bf16": dict(index=2, T=4096, H=7168, E=256, K=8, R=8, A=128, zero_pad=True,
                         fp8=False, gate="zipf", zipf_s=1.2, drop=0.0, max_tokens_per_rank=0),
    "fp8_dispatch": dict(index=3, T=4096, H=7168, E=256, K=8, R=8, A=128, zero_pad=True,
                         fp8=True, gate="zipf", zipf_s=1.2, drop=0.0, max_tokens_per_rank=0),
    "decode": dict(index=4, T=4096, H=7168, E=256, K=8, R=32, A=1, zero_pad=False, fp8=False,
                   gate="uniform", zipf_s=None, drop=0.1, max_tokens_per_rank=128),
    "large_prefill": dict(index=5, T=16384, H=7168, E=256, K=8, R=64, A=128, zero_pad=True,
                          fp8=False, gate="zipf", zipf_s=1.5, drop=0.0, max_tokens_per_rank=0),
}

HOT_SHARE_TARGET = 0.20   # two hot experts take ~20 % of pairs in the large-prefill gate
CALIBRATION = "large_prefill"


def config(name, **overrides):
    cfg = dict(WORKLOADS[name])
    cfg["name"] = name
    cfg["seed"] = 1000 + cfg["index"]
    cfg.update(overrides)
    return cfg


def _streams(seed):
    ss = np.random.SeedSequence(seed)
    return [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(4)]


def to_bf16_bits(f32):
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def _topk_sets_counts(scores, K, E):
    part = np.argpartition(-scores, K - 1, axis=1)[:, :K]
    return np.bincount(part.ravel(), minlength=E)


def _zipf_bias_shape(rng, E, s):
    perm = rng.permutation(E)
    rank = perm.astype(np.float64) + 1.0
    return -s * np.log(rank)


def _gate_noise(cfg, rng):
    T, E = cfg["T"], cfg["E"]
    if cfg["gate"] == "uniform":
        return rng.random((T, E))
    return rng.standard_normal((T, E))


def _gate_scores(cfg, rng, beta):
    noise = _gate_noise(cfg, rng)
    if cfg["gate"] == "uniform":
        return noise
    bias = _zipf_bias_shape(rng, cfg["E"], cfg["zipf_s"])
    return noise + beta * bias[None, :]


@functools.lru_cache(maxsize=None)
def zipf_beta():
    """Bias strength beta: bisection so the large-prefill gate's top-2 experts take 20 % of pairs."""
    cfg = config(CALIBRATION)
    g = _streams(cfg["seed"])[0]
    noise = _gate_noise(cfg, g)
    bias = _zipf_bias_shape(g, cfg["E"], cfg["zipf_s"])
    total = cfg["T"] * cfg["K"]

    def share(beta):
        counts = _topk_sets_counts(noise + beta * bias[None, :], cfg["K"], cfg["E"])
        return np.sort(counts)[-2:].sum() / total

    lo, hi = 0.0, 1.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if share(mid) < HOT_SHARE_TARGET:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def routing(cfg):
    """topk_idx int64 [T, K] and topk_weights fp32 [T, K] for a workload."""
    T, E, K = cfg["T"], cfg["E"], cfg["K"]
    g_gate, g_drop, _, _ = _streams(cfg["seed"])
    beta = zipf_beta() if cfg["gate"] == "zipf" else 0.0
    scores = _gate_scores(cfg, g_gate, beta)
    order = np.argsort(-scores, axis=1, kind="stable")[:, :K]
    topk_idx = order.astype(np.int64)
    sel = np.take_along_axis(scores, order, axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    topk_weights = (z / z.sum(axis=1, keepdims=True)).astype(np.float32)
    if cfg["drop"] > 0:
        mask = g_drop.random((T, K)) < cfg["drop"]
        topk_idx[mask] = -1
    return np.ascontiguousarray(topk_idx), np.ascontiguousarray(topk_weights)


def tokens(cfg, rows=None):
    """x: bf16 bits [T, H] drawn from N(0, 1).  ``rows`` limits to the first rows."""
    T = cfg["T"] if rows is None else rows
    g_x = _streams(cfg["seed"])[2]
    return to_bf16_bits(g_x.standard_normal((T, cfg["H"]), dtype=np.float32))


def expert_outputs(cfg, rows, seed_offset=0):
    """Expert outputs for combine: bf16 bits [rows, H], random sign and 7-bit
    mantissa, exponent uniform in [-7, 3] (magnitudes in [2^-7, 16))."""
    g_y = np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg["seed"], 4, seed_offset])))
    H = cfg["H"]
    # 16 random bits per value: bit 0 sign, bits 1-7 mantissa, bits 8-15 pick
    # the exponent (256 codes spread over the 11 exponents)
    expo_of = ((127 - 7 + np.arange(256) * 11 // 256) << 7).astype(np.uint16)
    out = np.empty((rows, H), np.uint16)
    step = 8192
    for r0 in range(0, rows, step):
        n = min(step, rows - r0)
        r = g_y.bit_generator.random_raw((n * H + 3) // 4).view(np.uint16)[:n * H].reshape(n, H)
        v = expo_of[r >> np.uint16(8)]
        v |= (r & np.uint16(1)) << np.uint16(15)
        v |= (r >> np.uint16(1)) & np.uint16(0x7F)
        out[r0:r0 + step] = v
    return out


def inputs(cfg, with_x=True):
    """All inputs of one workload as host numpy arrays."""
    idx, w = routing(cfg)
    out = dict(topk_idx=idx, topk_weights=w)
    if with_x:
        out["x"] = tokens(cfg)
    return out


def load_stats(topk_idx, E):
    """Realised load: max / mean expert load and the top-2 share of pairs."""
    v = topk_idx[topk_idx >= 0]
    counts = np.bincount(v, minlength=E)
    n = max(v.size, 1)
    return dict(pairs=int(v.size), max_over_mean=float(counts.max() / max(counts.mean(), 1e-9)),
                top2_share=float(np.sort(counts)[-2:].sum() / n),
                empty_experts=int((counts == 0).sum()))
