"""The N > 1 path of bench.py, on the CPU with world-size-2 `gloo` processes.

With several GPUs every rank runs its own replica of the single-GPU path (there
is no data-path collective); the process group only provides the barrier and
the max over ranks of the step time, and the job throughput sums the tokens of
all ranks.  These host-side pieces are exercised here without a GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        step_ms = [0.25, 0.40][rank]                 # rank 1 is the slower one
        m = bench.max_over_ranks(step_ms, dist, "cpu")
        value = bench.job_throughput(4096, world, m)
        dist.barrier()
        out.put((rank, m, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, q), nprocs=2, join=True, start_method="spawn")
    got = sorted(q.get(timeout=30) for _ in range(2))
    for rank, m, value in got:
        assert m == pytest.approx(0.40)                          # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 4096 / 0.40e-3)       # tokens of both ranks over that time


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.3, None, "cpu") == pytest.approx(0.3)
    assert bench.job_throughput(100, 1, 1.0) == pytest.approx(1e5)


@pytest.mark.slow
def test_reference_arm_under_torchrun_prints_one_line():
    """`bench.py --impl reference` launched as 2 ranks: rank 0 alone times the
    CPU oracle and prints the one JSON line; the other rank exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1", "--gpus", "2"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300,
                         env=dict(os.environ, OMP_NUM_THREADS="1"))
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["n_gpus"] == 2 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_algorithmic_bytes_accounting():
    """The bytes the roofline divides by, from the definitions: dispatch reads
    each token row once and writes every receive row (pairs and, with zero
    padding, the padding rows) plus the pair slots; combine reads one row per
    pair, writes one row per token and reads the slots and weights."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import workload
    cfg = workload.config("prefill_bf16")
    T, H, K, E, A = cfg["T"], cfg["H"], cfg["K"], cfg["E"], cfg["A"]
    cnt = np.full(E, 128, np.int64)
    cnt[:3] = [1, 129, 0]
    N = int(cnt.sum())
    Np = int(((cnt + A - 1) // A * A).sum())
    b = bench.algorithmic_bytes(cfg, cnt, A)
    assert (b["N"], b["Np"], b["pad_rows"]) == (N, Np, Np - N)
    # layout: topk_idx and weights read once, one slot written per entry, 12 B per receive row, E counts
    assert b["layout"] == T * K * (8 + 4 + 4) + Np * 12 + E * 8
    assert b["dispatch"] == T * 2 * H + Np * 2 * H + T * K * 4
    assert b["combine"] == N * 2 * H + T * 2 * H + T * K * 8
    fp8 = dict(cfg, fp8=True)
    assert bench.algorithmic_bytes(fp8, cnt, A)["dispatch"] == T * 2 * H + Np * (H + 4 * H // 128) + T * K * 4
    nopad = dict(cfg, zero_pad=False)
    assert bench.algorithmic_bytes(nopad, cnt, A)["dispatch"] == T * 2 * H + N * 2 * H + T * K * 4
    slab = bench.algorithmic_bytes(nopad, cnt, 1, slab=4096)
    assert slab["Np"] == E * 4096 and slab["dispatch"] == T * 2 * H + N * 2 * H + T * K * 4
    rank = bench.algorithmic_bytes_rank(cfg, rows=20000, N=N)
    assert rank["dispatch"] == T * 2 * H + 20000 * 2 * H + T * cfg["R"] * 4
    assert rank["combine"] == 20000 * 2 * H + T * 2 * H + T * cfg["R"] * 4


@pytest.mark.parametrize("form", ["expand", "rank", "ll"])
def test_reference_line_names_our_workload(form):
    """The reference arm prints the workload keys of `config` from the same
    function as our arm, with the oracle's own pair and receive-row counts."""
    import argparse
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import oracle
    import workload
    args = argparse.Namespace(workload="tiny", tokens=None, layout=form, steps=1, warmup=0)
    line = bench.run_reference(args, 0, 1)
    cfg = workload.config("tiny")
    inp = workload.inputs(cfg)
    lay = oracle.step_layout(inp, cfg, form)
    c = line["config"]
    assert line["impl"] == "reference" and c["workload"].startswith("tiny: T=128 H=256 E=16 top-4 R=2")
    assert c["pairs"] == int((inp["topk_idx"] >= 0).sum())
    assert c["recv_rows"] == int(lay["off"][-1])
    expect = bench.workload_config(cfg, form, 1, {"N": c["pairs"], "Np": c["recv_rows"], "pad_rows": c["pad_rows"]},
                                   inp["topk_idx"])
    assert c == expect                      # the same keys and values as our arm's config
    assert np.isfinite(line["value"]) and line["value"] > 0


def test_default_workload_is_the_largest_one_gpu_configuration(monkeypatch):
    """With no flags the bench times large_prefill (T = 16384, R = 64), the
    largest configuration that fits one GPU, and follows it with the others."""
    sys.path.insert(0, ROOT)
    import bench
    import workload
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    args = bench.parse()
    assert args.workload == "large_prefill" and args.per_workload and args.gpus == 1
    assert args.warmup >= 3
    cfg = bench.bench_config(args)
    assert max(workload.WORKLOADS, key=lambda n: workload.WORKLOADS[n]["T"]) == "large_prefill"
    assert (cfg["T"], cfg["H"], cfg["E"], cfg["K"], cfg["R"], cfg["A"]) == (16384, 7168, 256, 8, 64, 128)


@pytest.mark.parametrize("body,expect", [
    ('{"hbm_gbs": 6548.2}', (6548.2, "measured")),
    ('{"hbm_gbs": {"value": 6500}}', (6500.0, "measured")),
    ('{"hbm_gbs": {"gbs": 6400.5}}', (6400.5, "measured")),
    ('{"bf16_tflops": 1590}', (6650.0, "fallback")),
    ('{"hbm_gbs": null}', (6650.0, "fallback")),
    ('{"hbm_gbs": -1}', (6650.0, "fallback")),
    ('not json', (6650.0, "fallback")),
])
def test_measured_peaks_reader(tmp_path, monkeypatch, body, expect):
    """The HBM denominator comes from MEASURED_PEAKS.json when it holds a
    positive hbm_gbs (plain or under "value" / "gbs"), else the fallback."""
    import bench
    (tmp_path / "MEASURED_PEAKS.json").write_text(body)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == expect


def test_measured_peaks_absent(tmp_path, monkeypatch):
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (6650.0, "fallback")
