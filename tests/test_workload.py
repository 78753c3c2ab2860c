"""Self-checks of the seeded workload generator (the distribution-shape checks
that "DeepEP 测试目标 API 系统性参考" §5 lists for gate.py / test_gate.py)."""
import numpy as np
import pytest

import workload


@pytest.mark.parametrize("name", sorted(workload.WORKLOADS))
def test_routing_shape_and_determinism(name):
    cfg = workload.config(name)
    idx, w = workload.routing(cfg)
    idx2, w2 = workload.routing(cfg)
    assert np.array_equal(idx, idx2) and np.array_equal(w, w2)
    T, K, E = cfg["T"], cfg["K"], cfg["E"]
    assert idx.shape == (T, K) and idx.dtype == np.int64 and w.dtype == np.float32
    assert idx.min() >= -1 and idx.max() < E
    for t in range(0, T, max(1, T // 64)):          # no expert twice in one token
        row = idx[t][idx[t] >= 0]
        assert np.unique(row).size == row.size
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)           # best score first


def test_skewed_gate_hits_hot_share():
    cfg = workload.config("large_prefill")
    idx, _ = workload.routing(cfg)
    st = workload.load_stats(idx, cfg["E"])
    assert abs(st["top2_share"] - 0.20) <= 0.01
    cfg2 = workload.config("prefill_bf16")
    st2 = workload.load_stats(workload.routing(cfg2)[0], cfg2["E"])
    assert 0.02 < st2["top2_share"] < st["top2_share"]   # s = 1.2 is milder than s = 1.5


def test_decode_drop_fraction_and_uniform_load():
    cfg = workload.config("decode")
    idx, _ = workload.routing(cfg)
    frac = float((idx == -1).mean())
    assert abs(frac - 0.10) < 0.01
    st = workload.load_stats(idx, cfg["E"])
    assert st["max_over_mean"] < 1.5 and st["empty_experts"] == 0


def test_token_rows_are_bf16_normal():
    cfg = workload.config("tiny")
    x = workload.tokens(cfg)
    assert x.shape == (cfg["T"], cfg["H"]) and x.dtype == np.uint16
    f = (x.astype(np.uint32) << 16).view(np.float32)
    assert abs(f.mean()) < 0.02 and abs(f.std() - 1.0) < 0.02
    assert np.array_equal(x, workload.tokens(cfg))


def test_expert_outputs_range():
    cfg = workload.config("tiny")
    y = workload.expert_outputs(cfg, 64)
    f = np.abs((y.astype(np.uint32) << 16).view(np.float32))
    assert f.min() >= 2.0 ** -7 and f.max() < 16.0
    assert np.array_equal(y, workload.expert_outputs(cfg, 64))


@pytest.mark.parametrize("name,pairs,rows", [
    ("tiny", 512, 512),
    ("prefill_bf16", 32768, 56576),
    ("fp8_dispatch", 32768, 56576),
    ("decode", 29418, 29418),
    ("large_prefill", 131072, 153472),
])
def test_realised_workload_sizes(name, pairs, rows):
    """The seeded inputs are fixed: the pair and receive-row counts every
    reported figure was measured on (the oracle's layout of each workload)."""
    import oracle
    cfg = workload.config(name)
    inp = workload.inputs(cfg, with_x=False)
    lay = oracle.layout(inp["topk_idx"], inp["topk_weights"], cfg["E"], cfg["R"], cfg["A"])
    assert int((inp["topk_idx"] >= 0).sum()) == pairs
    assert int(lay["off"][-1]) == rows
