"""Benchmark: MoE dispatch + combine on one B200 (or N independent replicas).

One step = the whole hot path over one batch: ep_layout (one kernel),
ep_dispatch (with the fused FP8 cast for the FP8 workload) and ep_combine, on
the default workload "large_prefill", the largest one-GPU configuration:
T = 16384 tokens, H = 7168 bf16, 256 experts, top-8, R = 64 virtual ranks
(4 experts each), expert_alignment 128, zero padding, heavily skewed (Zipf
s = 1.5 bias, two hot experts take about 20 % of the pairs) gate, weighted
combine.  Inputs are seeded synthetic (workload/), resident in HBM before
timing; the combine input ("expert outputs") is the dispatched receive buffer
itself (identity experts).  After the headline, the same measurement runs on
every other workload (tiny, prefill_bf16, fp8_dispatch, decode) and is
reported under "per_workload" (one GPU only).

Timing: W warm-up steps, then K steps; before every step L2 is flushed by
writing a 256 MiB buffer (outside the timed events); each step is timed with
CUDA events on the launching stream, and per kernel as well.  Multi-GPU
(torchrun): every rank runs its own replica (the path is one GPU's HBM; no
data-path collective), the step time is the max over ranks, `value` sums the
tokens of all ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workload  # noqa: E402

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s vs B200 peak (1 GPU)"
FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="large_prefill", choices=sorted(workload.WORKLOADS))
    p.add_argument("--tokens", type=int, default=None,
                   help="override the workload's token count T (a multiple of its rank count)")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-per-workload", dest="per_workload", action="store_false",
                   help="time only the headline workload (by default the others follow it on one GPU)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--fused", action="store_true",
                   help="the single ep_layout_dispatch call instead of ep_layout + ep_dispatch")
    p.add_argument("--no-flush", dest="flush", action="store_false",
                   help="no L2 flush between steps (each step's inputs, x and the expert outputs, exceed L2)")
    p.add_argument("--no-graph", dest="graph", action="store_false",
                   help="launch the calls of every step instead of replaying one captured CUDA graph")
    p.add_argument("--layout", default="expand", choices=["expand", "rank", "ll"],
                   help="expand: one receive row per (token, k) pair (ep_layout); rank: one per (token, rank) "
                        "reached (ep_rank_layout) with V1's unweighted combine; ll: the low-latency fixed "
                        "slab of R * max_tokens rows per expert (ep_ll_layout)")
    return p.parse_args()


def bench_config(args):
    """The workload's configuration, with T overridden by --tokens."""
    cfg = workload.config(args.workload)
    if args.tokens is not None:
        if args.tokens < 0 or args.tokens % cfg["R"]:
            raise SystemExit("--tokens must be a non-negative multiple of R = %d" % cfg["R"])
        cfg = dict(cfg, T=args.tokens)
    return cfg


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        v = d["hbm_gbs"]
        if isinstance(v, dict):   # {"value": ...} or {"gbs": ...}
            v = v.get("value", v.get("gbs"))
        v = float(v)
        if not v > 0:
            raise ValueError("hbm_gbs")
        return v, "measured"
    except (OSError, KeyError, ValueError, TypeError):
        return 6650.0, "fallback"


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, wl):
    """DRAM bytes (read + write) per launch from the committed ncu capture
    (profiles/traffic.json), if it was taken on the current kernel sources;
    else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    rec = d.get("%s@%s" % (kernel, wl))
    try:
        if not rec or rec.get("source_sha") != source_hash(rec["sources"]):
            return None
    except OSError:
        return None
    return rec.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------
# multi-rank host logic: every rank runs its own replica
# --------------------------------------------------------------------------
def max_over_ranks(x, dist, device):
    """The max of a per-rank value over all ranks (step times are taken as the
    slowest rank's); the identity on one rank."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, ms_per_step):
    """Whole-job tokens/s: the tokens of all ranks over the (max) step time."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        rows = [r for r in self.rows if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------
# algorithmic bytes (the minimum each step must move)
# --------------------------------------------------------------------------
def algorithmic_bytes(cfg, cnt, A, slab=0):
    T, H, K, E = cfg["T"], cfg["H"], cfg["K"], cfg["E"]
    N = int(cnt.sum())
    Np = E * slab if slab else int(((cnt + A - 1) // A * A).sum())
    pad = (Np - N) if cfg["zero_pad"] else 0
    nb = H // 128
    out_row = (H + 4 * nb) if cfg["fp8"] else 2 * H
    layout_b = T * K * (8 + 4 + 4) + Np * 12 + E * 8     # idx and weights read, slots written, row maps, counts
    dispatch_b = T * 2 * H + (N + pad) * out_row + T * K * 4
    combine_b = N * 2 * H + T * K * 8 + T * 2 * H
    return dict(layout=layout_b, dispatch=dispatch_b, combine=combine_b, N=N, Np=Np, pad_rows=Np - N)


def algorithmic_bytes_rank(cfg, rows, N):
    """The per-token-per-rank form: `rows` receive rows, one per (token, rank) reached."""
    T, H, K, E, R = cfg["T"], cfg["H"], cfg["K"], cfg["E"], cfg["R"]
    nb = H // 128
    out_row = (H + 4 * nb) if cfg["fp8"] else 2 * H
    # idx and weights read, is_token_in_rank + token_slot, recv_src + recv_topk_idx/weights, counts
    layout_b = T * K * 12 + T * R * 5 + rows * (4 + K * 12) + E * 8 + R * 8
    dispatch_b = T * 2 * H + rows * out_row + T * R * 4
    combine_b = rows * 2 * H + T * 2 * H + T * R * 4
    return dict(layout=layout_b, dispatch=dispatch_b, combine=combine_b, N=N, Np=rows, pad_rows=0)


def l2_statement(cfg, nbytes):
    """How the workload relates to the 126 MB L2: a property of the work, the
    same for both arms (the GPU arm's own flush is reported beside `config`)."""
    read_mb = (cfg["T"] + nbytes["Np"] - nbytes["pad_rows"]) * cfg["H"] * 2 / 1e6
    if read_mb > 126:
        return "inputs larger than L2: each step reads x and the expert-output rows, %.0f MB > 126 MB" % read_mb
    return "inputs fit in L2 (%.1f MB per step)" % read_mb


def workload_config(cfg, form, world, nbytes, topk_idx):
    """The `config` keys that name the workload; both arms print exactly these,
    so the reference line describes exactly the work of ours."""
    T, H, E, K, R, A = (cfg[k] for k in ("T", "H", "E", "K", "R", "A"))
    M = cfg["max_tokens_per_rank"] or T // R
    shape = {"expand": "",
             "rank": " layout=per-rank (one row per token and rank reached, unweighted combine)",
             "ll": " layout=ll (fixed slab of R*%d rows per expert)" % M}[form]
    return {"workload": "%s: T=%d H=%d E=%d top-%d R=%d align=%d zero_pad=%s%s%s" % (
                cfg["name"], T, H, E, K, R, A, cfg["zero_pad"], " fp8-cast" if cfg["fp8"] else "", shape),
            "global_batch": T * world, "parallelism": "replicas x%d (R=%d virtual ranks per GPU)" % (world, R),
            "pairs": nbytes["N"], "recv_rows": nbytes["Np"], "pad_rows": nbytes["pad_rows"],
            "load": workload.load_stats(topk_idx, E), "l2": l2_statement(cfg, nbytes)}


def form_bytes(cfg, form, cnt_or_rows, n_pairs):
    """Algorithmic bytes of one step of `form` on `cfg`: cnt_or_rows is the
    per-expert pair counts (expand, ll) or the receive-row count (rank)."""
    if form == "rank":
        return algorithmic_bytes_rank(cfg, cnt_or_rows, n_pairs)
    if form == "ll":
        return algorithmic_bytes(cfg, cnt_or_rows, 1, slab=cfg["R"] * (cfg["max_tokens_per_rank"] or
                                                                       cfg["T"] // cfg["R"]))
    return algorithmic_bytes(cfg, cnt_or_rows, cfg["A"])


# --------------------------------------------------------------------------
# our implementation
# --------------------------------------------------------------------------
class Step:
    """One workload set up on the device: inputs resident in HBM, the handle,
    the receive and output buffers, and the calls of one step."""

    def __init__(self, args, cfg, ep, torch, dev):
        self.args, self.cfg, self.ep, self.torch, self.dev = args, cfg, ep, torch, dev
        self.inp = inp = workload.inputs(cfg)
        T, H, K, E, R, A = cfg["T"], cfg["H"], cfg["K"], cfg["E"], cfg["R"], cfg["A"]
        self.idx = torch.from_numpy(inp["topk_idx"]).to(dev)
        self.w = torch.from_numpy(inp["topk_weights"]).to(dev)
        self.x = torch.from_numpy(inp["x"].view(np.int16)).to(dev).view(torch.bfloat16)
        self.form = args.layout
        self.per_rank = self.form == "rank"
        self.slab = self.form == "ll"
        self.M = cfg["max_tokens_per_rank"] or T // R
        if self.form != "expand" and args.fused:
            raise SystemExit("--fused applies to the expand layout only")
        if self.per_rank:
            self.lay = ep.RankLayout(T, K, E, R, A, dev)
        elif self.slab:
            self.lay = ep.ll_layout(self.idx, self.w, E, R, self.M)
        else:
            self.lay = ep.Layout(T, K, E, R, A, dev, num_max_tokens_per_rank=cfg["max_tokens_per_rank"])
        self.cw = None if self.per_rank else self.w          # V1's combine is a plain sum over the ranks
        cap = self.lay.capacity
        self.fp8 = fp8 = cfg["fp8"]
        self.recv = torch.empty((cap, H), dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16, device=dev)
        self.recv_s = torch.empty((cap, H // 128), dtype=torch.float32, device=dev) if fp8 else None
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        # expert outputs for combine: identity experts (bf16), or seeded outputs for FP8
        self.do_layout(self.idx, self.w)
        self.dispatch()
        torch.cuda.synchronize(dev)
        if fp8:
            self.y = torch.from_numpy(workload.expert_outputs(cfg, cap).view(np.int16)).to(dev).view(torch.bfloat16)
        else:
            self.y = self.recv.clone()
        if self.per_rank:
            self.nbytes = form_bytes(cfg, "rank", self.lay.num_recv_rows(), int((self.idx >= 0).sum()))
        else:
            self.nbytes = form_bytes(cfg, self.form, self.lay.num_recv_tokens_per_expert.cpu().numpy(), None)

    def dispatch(self):
        cfg = self.cfg
        if self.fp8:
            self.ep.dispatch(self.lay, self.x, cast_to_fp8=True, do_zero_padding=cfg["zero_pad"], out=self.recv,
                             out_scales=self.recv_s)
        else:
            self.ep.dispatch(self.lay, self.x, do_zero_padding=cfg["zero_pad"], out=self.recv)

    def do_layout(self, d_idx, d_w):
        cfg, ep = self.cfg, self.ep
        if self.per_rank:
            ep.rank_layout(d_idx, d_w, cfg["E"], cfg["R"], cfg["A"], out=self.lay)
        elif self.slab:
            ep.ll_layout(d_idx, d_w, cfg["E"], cfg["R"], self.M, out=self.lay)
        else:
            ep.layout(d_idx, d_w, cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"], out=self.lay)

    def step(self, evs=None):
        cfg, ep, stream = self.cfg, self.ep, self.stream
        if evs:
            evs[0].record(stream)
        if not self.args.fused:
            self.do_layout(self.idx, self.w)
            if evs:
                evs[1].record(stream)
            self.dispatch()
        else:
            ep.layout_dispatch(self.idx, self.w, self.x, cfg["E"], cfg["R"], cfg["A"], cfg["max_tokens_per_rank"],
                               cast_to_fp8=self.fp8, do_zero_padding=cfg["zero_pad"], out_layout=self.lay,
                               out=self.recv, out_scales=self.recv_s)
            if evs:
                evs[1].record(stream)
        if evs:
            evs[2].record(stream)
        ep.combine(self.lay, self.y, self.cw, out=self.out)
        if evs:
            evs[3].record(stream)

    def check(self):
        """Device status clean; with identity experts and weights summing to one,
        combine(dispatch(x)) gives x back."""
        torch = self.torch
        torch.cuda.synchronize(self.dev)
        code, flags = self.ep.get_status(self.lay)
        assert code == 0, "device status %d (flags %d)" % (code, flags)
        if not self.fp8 and self.cfg["drop"] == 0 and not self.per_rank:
            has = (self.idx >= 0).any(dim=1)
            assert torch.equal(self.out[has].float(), self.x[has].float()), "combine(dispatch(x)) != x"


def time_steps(st, args, flush, dist, dev, clocks=None):
    """W warm-up steps, then K timed steps (one event pair around each; no
    events between the kernels), then K more with events between the calls
    for the per-kernel split.  Returns the timings in ms."""
    torch = st.torch
    for _ in range(args.warmup):
        flush.zero_()
        st.step()
    st.check()
    # optionally one step captured as a CUDA graph (the calls allocate nothing
    # and only enqueue work, so they capture as they are)
    run_step, graph = st.step, None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            st.step()
        torch.cuda.synchronize(dev)
        for _ in range(3):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize(dev)
        run_step = graph.replay
    stream = st.stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.start()
        time.sleep(0.3)
    wall0 = time.perf_counter()
    for i in range(args.steps):
        if args.flush:
            flush.zero_()
        evs[i][0].record(stream)
        run_step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    if dist:
        dist.barrier()
    clock_info = clocks.stop() if clocks else None
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    # per-kernel breakdown: the same K steps again with events between the kernels
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        if args.flush:
            flush.zero_()
        st.step(evk[i])
    torch.cuda.synchronize(dev)
    st.check()
    per = np.array([[evk[i][j].elapsed_time(evk[i][j + 1]) for j in range(3)] for i in range(args.steps)])
    del graph
    return dict(ms_mean=float(np.mean(step_ms)), ms_median=float(np.median(step_ms)),
                kernel_ms=per.mean(axis=0), wall=wall, clocks=clock_info)


def kernel_summary(st, args, k_ms, peak):
    """Per-kernel times, the dominant kernel's achieved bandwidth and its roofline fraction."""
    nb = st.nbytes
    if not args.fused:
        top_kernel = "dispatch_cast_kernel" if st.fp8 else "dispatch_copy_kernel"
        top_bytes, top_ms = nb["dispatch"], k_ms[1]
        kernels_us = {"layout": round(k_ms[0] * 1e3, 2), "dispatch": round(k_ms[1] * 1e3, 2)}
    else:
        top_kernel = "layout_kernel+dispatch_cast_kernel" if st.fp8 else "layout_kernel+dispatch_copy_kernel"
        top_bytes, top_ms = nb["layout"] + nb["dispatch"], k_ms[0] + k_ms[1]
        kernels_us = {"layout_dispatch": round(top_ms * 1e3, 2)}
    kernels_us["combine"] = round(k_ms[2] * 1e3, 2)
    disp_gbs = top_bytes / (top_ms * 1e-3) / 1e9
    return dict(top_kernel=top_kernel, top_bytes=top_bytes, disp_gbs=disp_gbs, kernels_us=kernels_us,
                combine_gbs=nb["combine"] / (k_ms[2] * 1e-3) / 1e9, frac=disp_gbs / peak)


def step_bytes(nb):
    return nb["layout"] + nb["dispatch"] + nb["combine"]


def per_workload_entry(st, args, tm, peak):
    """One line of `per_workload`: a whole-step and per-kernel summary."""
    ks = kernel_summary(st, args, tm["kernel_ms"], peak)
    ms = tm["ms_mean"]
    total = step_bytes(st.nbytes)
    return {"workload": workload_config(st.cfg, args.layout, 1, st.nbytes, st.inp["topk_idx"])["workload"],
            "ms_per_step": round(ms, 5), "ms_per_step_median": round(tm["ms_median"], 5),
            "tokens_per_s": round(st.cfg["T"] / (ms * 1e-3), 1),
            "hbm_gbs": round(total / (ms * 1e-3) / 1e9, 1),
            "hbm_frac_of_measured": round(total / (ms * 1e-3) / 1e9 / peak, 4),
            "hbm_frac_of_nominal_8tbs": round(total / (ms * 1e-3) / 1e9 / 8000.0, 4),
            "algorithmic_bytes_per_step": total,
            "kernels_us": ks["kernels_us"],
            "dispatch": {"kernel": ks["top_kernel"], "gbs": round(ks["disp_gbs"], 1), "frac": round(ks["frac"], 4)},
            "combine_gbs": round(ks["combine_gbs"], 1),
            "gpu_launches_per_step": 3}


def run_ours(args, rank, world, local_rank):
    import torch
    import combine_ep_layout_11_b200 as ep
    from combine_ep_layout_11_b200 import build as lib_build
    if rank == 0 or not os.path.exists(lib_build.LIB):
        lib_build.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    cfg = bench_config(args)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    st = Step(args, cfg, ep, torch, dev)
    T, H = cfg["T"], cfg["H"]
    clocks = ClockSampler(local_rank) if (rank == 0 and not args.no_clocks) else None
    tm = time_steps(st, args, flush, dist, dev, clocks)
    ms_per_step = max_over_ranks(tm["ms_mean"], dist, dev)
    ms_median = max_over_ranks(tm["ms_median"], dist, dev)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, ep, torch, dev, st.inp, cfg, st.lay, st.y, st.fp8, st.recv, st.recv_s, flush,
                      st.do_layout, st.per_rank)
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dist, dev)
        e2e["copy_ms_per_step"] = max_over_ranks(e2e["copy_ms_per_step"], dist, dev)

    if rank != 0:
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return None

    peak, peak_kind = measured_peaks()
    nbytes, fp8 = st.nbytes, st.fp8
    payload_rows = nbytes["Np"] - nbytes["pad_rows"]
    ks = kernel_summary(st, args, tm["kernel_ms"], peak)
    total_bytes = step_bytes(nbytes)
    kernels_us = dict(ks["kernels_us"], note="second pass with events between the calls")
    value = job_throughput(T, world, ms_per_step)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8-e4m3/bf16" if fp8 else "bf16",
        "data": "synthetic (seeded; workload/ generator, seed %d)" % cfg["seed"],
        "config": workload_config(cfg, args.layout, world, nbytes, st.inp["topk_idx"]),
        "l2_flush": ("a 256 MiB write before every step, outside the timed events" if args.flush else
                     "none (the step's inputs exceed L2)"),
        "launch": "one CUDA graph per step" if args.graph else "stream launches with programmatic dependent launch",
        "ms_per_step_median": round(ms_median, 5),
        # the count_bytes convention: one row copy in dispatch and one row read in
        # combine per receive row that holds data
        "payload_gbs": round(payload_rows * ((H + 4 * (H // 128) if fp8 else 2 * H) + 2 * H)
                             / (ms_per_step * 1e-3) / 1e9, 1),
        "hbm_gbs": round(total_bytes / (ms_per_step * 1e-3) / 1e9, 1),
        "hbm_frac_of_measured": round(total_bytes / (ms_per_step * 1e-3) / 1e9 / peak, 4),
        "hbm_frac_of_nominal_8tbs": round(total_bytes / (ms_per_step * 1e-3) / 1e9 / 8000.0, 4),
        "algorithmic_bytes_per_step": total_bytes,
        "kernels_us": kernels_us,
        "kernels_gbs": {"dispatch": round(ks["disp_gbs"], 1), "combine": round(ks["combine_gbs"], 1)},
        "roofline": {"bound": "hbm", "kernel": ks["top_kernel"],
                     "achieved": round(ks["disp_gbs"], 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(ks["frac"], 4),
                     "traffic": ncu_traffic(ks["top_kernel"], cfg["name"] + ("" if args.layout == "expand"
                                                                             else "/" + args.layout)),
                     "algorithmic_bytes_per_launch": ks["top_bytes"]},
        "gpu_launches": args.steps * 3,
        "wall_s_timed_region": round(tm["wall"], 4),
    }
    if tm["clocks"]:
        line["clocks"] = tm["clocks"]
    if e2e:
        line["e2e"] = {"value": round(job_throughput(T, world, e2e["ms_per_step"]), 1), "unit": "tokens/s",
                       "ms_per_step": round(e2e["ms_per_step"], 4),
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "how": "%d steps through the public API from pinned host buffers: every step uploads "
                              "topk_idx, topk_weights and x and downloads the combined output; the expert "
                              "outputs (the combine input) stay resident on the device, as a GPU expert layer "
                              "produces them there; uploads, calls and downloads pipelined over three streams, "
                              "timed from the first upload to the last download; no L2 flush (each step moves "
                              "more than L2 holds)" % e2e["steps"],
                       "copy_bound": {"ms_per_step": round(e2e["copy_ms_per_step"], 4),
                                      "frac": round(e2e["copy_ms_per_step"] / e2e["ms_per_step"], 4),
                                      "gbs_per_direction": round(max(e2e["h2d"], e2e["d2h"]) /
                                                                 (e2e["copy_ms_per_step"] * 1e6), 1),
                                      "how": "the same uploads and downloads alone (no calls), both "
                                             "directions at once: the PCIe ceiling of this leg; frac = "
                                             "that time over the leg's"}}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, st.inp, args.layout)
    if world == 1 and args.per_workload and args.tokens is None:
        # every other workload, same measurement, one at a time (buffers freed in between)
        del st, e2e
        torch.cuda.empty_cache()
        entries = {}
        for name in sorted(workload.WORKLOADS, key=lambda n: workload.WORKLOADS[n]["index"]):
            if name == cfg["name"]:
                continue
            other = Step(args, workload.config(name), ep, torch, dev)
            entries[name] = per_workload_entry(other, args, time_steps(other, args, flush, None, dev), peak)
            del other
            torch.cuda.empty_cache()
        line["per_workload"] = entries
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return line


def run_e2e(args, ep, torch, dev, inp, cfg, lay, y, fp8, recv, recv_s, flush, do_layout, per_rank):
    """Same steps through the public API with host buffers: every step copies
    its inputs from pinned host memory, runs the calls and copies the combined
    output back.  The steps are pipelined over three streams, as a serving
    loop would run them: step i+1's inputs go up and step i-1's output comes
    down while step i computes (double-buffered device inputs and outputs; the
    calls of consecutive steps stay in order on one stream).  Timed from the
    first upload to the last download."""
    T, H = cfg["T"], cfg["H"]
    h_idx = torch.from_numpy(inp["topk_idx"]).pin_memory()
    h_w = torch.from_numpy(inp["topk_weights"]).pin_memory()
    h_x = torch.from_numpy(inp["x"].view(np.int16)).pin_memory()
    h_out = [torch.empty((T, H), dtype=torch.int16).pin_memory() for _ in range(2)]
    d_idx = [torch.empty_like(h_idx, device=dev) for _ in range(2)]
    d_w = [torch.empty_like(h_w, device=dev) for _ in range(2)]
    d_x = [torch.empty_like(h_x, device=dev) for _ in range(2)]
    d_out = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    s_up, s_comp, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    steps = max(3, min(args.steps, 20))

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_comp[b])       # step i-2 has finished reading buffer b
                d_idx[b].copy_(h_idx, non_blocking=True)
                d_w[b].copy_(h_w, non_blocking=True)
                d_x[b].copy_(h_x, non_blocking=True)
                ev_up[b].record(s_up)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_up[b])
                if i >= 2:
                    s_comp.wait_event(ev_down[b])     # step i-2's output has left buffer b
                xb = d_x[b].view(torch.bfloat16)
                if args.fused:
                    ep.layout_dispatch(d_idx[b], d_w[b], xb, cfg["E"], cfg["R"], cfg["A"],
                                       cfg["max_tokens_per_rank"], cast_to_fp8=fp8,
                                       do_zero_padding=cfg["zero_pad"], out_layout=lay, out=recv, out_scales=recv_s)
                else:
                    do_layout(d_idx[b], d_w[b])
                    ep.dispatch(lay, xb, cast_to_fp8=fp8, do_zero_padding=cfg["zero_pad"], out=recv,
                                out_scales=recv_s)
                ep.combine(lay, y, None if per_rank else d_w[b], out=d_out[b])
                ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_comp[b])
                h_out[b].copy_(d_out[b].view(torch.int16), non_blocking=True)
                ev_down[b].record(s_down)

    run(2)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    run(steps)
    s_down.wait_stream(s_comp)
    e1.record(s_down)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    assert torch.equal(h_out[(steps - 1) % 2], d_out[(steps - 1) % 2].view(torch.int16).cpu())
    e2e_ms = e0.elapsed_time(e1) / steps

    # the ceiling of this leg: the same uploads and downloads with no calls,
    # both directions at once on their streams
    def copies(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_up):
                d_idx[b].copy_(h_idx, non_blocking=True)
                d_w[b].copy_(h_w, non_blocking=True)
                d_x[b].copy_(h_x, non_blocking=True)
            with torch.cuda.stream(s_down):
                h_out[b].copy_(d_out[b].view(torch.int16), non_blocking=True)

    copies(2)
    torch.cuda.synchronize(dev)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(s_up)
    s_down.wait_event(c0)
    copies(steps)
    s_down.wait_stream(s_up)
    c1.record(s_down)
    c1.synchronize()
    h2d = h_idx.numel() * 8 + h_w.numel() * 4 + h_x.numel() * 2
    return {"ms_per_step": e2e_ms, "h2d": int(h2d), "d2h": int(h_out[0].numel() * 2),
            "steps": steps, "copy_ms_per_step": c0.elapsed_time(c1) / steps}


# --------------------------------------------------------------------------
# CPU oracle: the baseline leg and the reference arm
# --------------------------------------------------------------------------
def oracle_step_inputs(cfg, inp, form="expand"):
    import oracle
    lay = oracle.step_layout(inp, cfg, form)
    y = oracle.dispatch_rows(inp["x"], lay, cfg["zero_pad"]) if not cfg["fp8"] else \
        workload.expert_outputs(cfg, int(lay["off"][-1]))
    return dict(inp, y=y)


def time_oracle(cfg, inp, budget_s=10.0, min_steps=1, max_steps=None, form="expand"):
    import oracle
    full = oracle_step_inputs(cfg, inp, form)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.step(full, cfg, form)
        n += 1
        el = time.perf_counter() - t0
        if (n >= min_steps and el >= budget_s) or (max_steps and n >= max_steps):
            return n, el


def cpu_baseline(cfg, inp, form="expand"):
    n, el = time_oracle(cfg, inp, budget_s=10.0, form=form)
    return {"value": round(cfg["T"] * n / el, 1), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "%d full step(s) of the %s workload (layout, dispatch%s, combine), single-threaded C, "
                      "%d host cores present" % (n, cfg["name"], " with cast" if cfg["fp8"] else "",
                                                 os.cpu_count() or 0)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cfg = bench_config(args)
    inp = workload.inputs(cfg)
    form = args.layout
    full = oracle_step_inputs(cfg, inp, form)
    import oracle
    olay = oracle.step_layout(inp, cfg, form)
    if form == "rank":
        nbytes = form_bytes(cfg, form, int(olay["off"][-1]), int((inp["topk_idx"] >= 0).sum()))
    else:
        nbytes = form_bytes(cfg, form, olay["cnt"], None)
    for _ in range(args.warmup):
        oracle.step(full, cfg, form)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.step(full, cfg, form)
        ts.append(time.perf_counter() - t0)
    ms = float(np.mean(ts)) * 1e3
    v = round(cfg["T"] / (ms * 1e-3), 1)
    return {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8-e4m3/bf16" if cfg["fp8"] else "bf16",
            "data": "synthetic (seeded; workload/ generator, seed %d)" % cfg["seed"],
            "config": workload_config(cfg, form, world, nbytes, inp["topk_idx"]),
            "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": "the full %s workload per step (single-threaded C oracle)" % cfg["name"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world, local_rank)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
