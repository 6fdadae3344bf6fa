"""Benchmark: the router verify window (GEMV over a 2.6 MB weight + top-10) on B200.

One step = one pass of the router hot path over one batch: for each window
size m in (1, 2, 4, 8, 16), A[m,2560] bf16 x W_r[2560,512] bf16 -> fp32 logits
(weight streamed once) -> per-row top-10.  That is 31 rows per step.  The
reported value is the fused form, router_gemv_topk's default (one launch per
window: the GEMV with the top-k as its tail); the two-launch form
(MR_ROUTER_TWO_LAUNCH: the GEMV kernel, then the top-k kernel) is timed over
the same K steps and printed beside it.  The weight comes from a
rotating pool of copies larger than twice the L2, so every launch reads it
from HBM.

Printed (rank 0, one JSON line): us_per_row over the whole step (lower is
better), the per-m curve (us_per_row, GB/s, the batching speedup
us_per_row(1)/us_per_row(8)), the GEMV roofline against the measured HBM copy
bandwidth, an end-to-end number through the public API with host buffers, the
GEMM TFLOP/s sweep on the prompt-chunk shapes, the CPU oracle as a baseline,
and the SM clocks seen during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --profile-case gemv|topk|gemm|...   # a few launches, for ncu
    python bench.py --selector-study                # every GEMM tile on every chunk shape
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WINDOWS = (1, 2, 4, 8, 16)
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e nominal bandwidth; fractions are also given against the measured copy
K_ROUTER, N_ROUTER, TOPK = 2560, 512, 10
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def roofline_time_us(nbytes: float, gbps: float) -> float:
    """Time in microseconds to move ``nbytes`` at ``gbps`` GB/s (1 GB = 1e9 B)."""
    return nbytes / (gbps * 1e9) * 1e6


def gemv_bytes(m: int, n: int, k: int) -> int:
    """Algorithmic HBM bytes of one GEMV call: W once, A once, C once."""
    return n * k * 2 + m * k * 2 + m * n * 4


def router_bytes(m: int) -> int:
    """Algorithmic HBM bytes of one fused router window: W once, A once, and
    the top-k indices and values (the logits are an intermediate)."""
    return N_ROUTER * K_ROUTER * 2 + m * K_ROUTER * 2 + m * TOPK * 8


def step_rows() -> int:
    return sum(WINDOWS)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# Source files whose change invalidates a recorded ncu traffic figure.
KERNEL_SOURCES = {
    "gemv_router": ("mrgemv.cu", "common.cuh", "topk_core.cuh"),
    "router_fused": ("mrgemv.cu", "common.cuh", "topk_core.cuh"),
    "gemm": ("gemm_f16.cu", "common.cuh"),
}


def _code_only(text: str) -> str:
    """Source text without comments and blank-line or indentation differences,
    so that an edit of comments alone keeps a recorded measurement valid."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.strip() for line in text.splitlines() if line.strip())


def kernel_source_hash(kernel: str = "gemv_router") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "verify_weight_streaming_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        entry = rec[kernel]
        if entry.get("source_hash") != kernel_source_hash(kernel):
            return None
        return float(entry["dram_bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""
        return False

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid not in parts[0]:
                continue
            rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ------------------------------------------------------------------ distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------- oracle side

def oracle_router_step(a16, w16, n_cols=None):
    """One router step on the CPU oracle: fp64 product, fp32 logits, top-10 per row.

    ``n_cols`` < 512 runs the step on the first n_cols weight columns only (a
    bounded sample of the same workload)."""
    import numpy as np
    import oracle
    w = w16 if n_cols is None else w16[:n_cols]
    for m in WINDOWS:
        c64, _ = oracle.matmul(a16[:m], "bf16", w, "bf16")
        oracle.topk(c64.astype(np.float32), min(TOPK, w.shape[0]))


def run_reference(args, world, rank, budget_s: float = 150.0):
    """The reference arm: the CPU oracle, as it stands, on this host's cores.

    Each step is a column sample of the router step sized so that warm-up plus
    K steps take about ``budget_s`` seconds; the value is scaled to full rows."""
    if rank != 0:
        return None
    import oracle
    import synth
    a16, w16 = synth.router(16)
    oracle.default()
    t0 = time.perf_counter()
    oracle_router_step(a16, w16)
    full = time.perf_counter() - t0
    frac = min(1.0, budget_s / max(1e-9, full * (args.steps + args.warmup)))
    n_cols = max(TOPK, int(N_ROUTER * frac))
    for _ in range(args.warmup):
        oracle_router_step(a16, w16, n_cols)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_router_step(a16, w16, n_cols)
    dt = time.perf_counter() - t0
    scale = n_cols / N_ROUTER
    us_per_row = dt * 1e6 / (args.steps * step_rows() * scale)
    line = {
        "impl": "reference", "metric": "us_per_row", "value": us_per_row, "unit": "us/row",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps / scale, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": us_per_row, "unit": "us/row", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"each step: windows m=1,2,4,8,16 on the first {n_cols} of 512 "
                                   f"weight columns (k=2560) + top-10, scaled to full rows"},
        "e2e": {"value": us_per_row, "unit": "us/row", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def workload_config():
    return {"workload": "router verify window: A[m,2560] bf16 x W_r[2560,512] bf16 (2.6 MB) -> "
                        "fp32 logits -> per-row top-10; m in (1,2,4,8,16) per step",
            "rows_per_step": step_rows(), "k": K_ROUTER, "n": N_ROUTER, "topk": TOPK,
            "l2": "weights rotated over a pool of copies > 2x L2 (cold HBM reads)",
            "parallelism": "replicas (independent windows per GPU)"}


# -------------------------------------------------------------------- GPU arm

class RouterBench:
    def __init__(self, device):
        import numpy as np
        import torch
        import synth
        import verify_weight_streaming_b200 as mr
        self.torch, self.mr, self.np = torch, mr, np
        self.device = device
        props = torch.cuda.get_device_properties(device)
        self.l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
        a16, w16 = synth.router(16)
        self.a16, self.w16 = a16, w16
        wbytes = w16.nbytes
        self.pool = max(2 * len(WINDOWS), int(math.ceil(2.2 * self.l2 / wbytes)))
        w = torch.from_numpy(w16.view(np.int16)).to(device)
        self.W = [w.clone() for _ in range(self.pool)]
        self.A = torch.from_numpy(a16.view(np.int16)).to(device)
        self.C = {m: torch.empty((m, N_ROUTER), dtype=torch.float32, device=device) for m in WINDOWS}
        self.idx = {m: torch.empty((m, TOPK), dtype=torch.int32, device=device) for m in WINDOWS}
        self.val = {m: torch.empty((m, TOPK), dtype=torch.float32, device=device) for m in WINDOWS}
        self.stream = torch.cuda.Stream(device)
        self.cursor = 0
        nbytes = mr.router_gemv_topk_workspace_bytes(16, N_ROUTER, False)
        self.ws = torch.zeros((nbytes + 3) // 4, dtype=torch.int32, device=device)

    def _next_w(self):
        w = self.W[self.cursor % self.pool]
        self.cursor += 1
        return w

    def step(self, flags, fused=True):
        """One router step: for each window size, GEMV + top-10 in one
        router_gemv_topk call (one fused launch, or the GEMV kernel then the
        top-k kernel with MR_ROUTER_TWO_LAUNCH)."""
        mr = self.mr
        for m in WINDOWS:
            mr.router_gemv_topk(self.A[:m], self._next_w(), TOPK, self.idx[m], self.val[m],
                                workspace=self.ws, flags=flags if fused else flags | mr.MR_ROUTER_TWO_LAUNCH)

    def capture_steps(self, count, flags, fused=True):
        """One CUDA graph per step, each with its own slice of the weight pool."""
        torch = self.torch
        graphs = []
        with torch.cuda.stream(self.stream):
            self.step(flags, fused)  # warm the launch path outside capture
        torch.cuda.synchronize()
        for _ in range(count):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.step(flags, fused)
            graphs.append(g)
        return graphs

    def time_graphs(self, graphs, reps):
        torch = self.torch
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            start.record(self.stream)
            for i in range(reps):
                graphs[i % len(graphs)].replay()
            end.record(self.stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end) * 1e3  # us


def run_gpu(args, world, rank, local):
    import numpy as np
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    import verify_weight_streaming_b200 as mr

    hbm_peak, tf_peak, tf_sus, peak_kind = load_peaks()
    rb = RouterBench(device)
    flags = 0 if args.no_pdl else mr.MR_GEMV_PDL
    steps_per_cycle = max(1, rb.pool // len(WINDOWS))
    # Two forms of the router step give identical outputs: one fused launch
    # per window (the API's default) and two launches (the GEMV kernel, then
    # the top-k kernel).  `value` is always the fused form; the two-launch
    # form is timed over the same K steps and printed beside it.
    forms = {"fused": rb.capture_steps(steps_per_cycle, flags, fused=True),
             "two_launch": rb.capture_steps(steps_per_cycle, flags, fused=False)}
    for g in forms.values():
        rb.time_graphs(g, max(args.warmup, 3))
    assert mr.mr_poll_errors() == 0

    props = torch.cuda.get_device_properties(device)
    uuid = str(getattr(props, "uuid", "")) or None
    form_us = {}
    clocks = {}
    for name, graphs in forms.items():
        # ---- timed region: exactly K steps
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(uuid) as clk:
            elapsed_us = rb.time_graphs(graphs, args.steps)
            # A short K-step region gets too few nvidia-smi samples: repeat the
            # same K steps (not part of the value) until ~1.5 s of load is sampled.
            extra = []
            while sum(extra) + elapsed_us < 1.5e6 and len(extra) < 5000 and not args.quick:
                extra.append(rb.time_graphs(graphs, args.steps))
        torch.cuda.synchronize()
        barrier(world)
        form_us[name] = max_over_ranks(elapsed_us, world, device)
        clocks[name] = clk.summary()
        clocks[name]["sampled_over_us"] = elapsed_us + sum(extra)
    errs = mr.mr_poll_errors()
    best_form = "fused"
    elapsed_max = form_us[best_form]
    # whole-job time per row: all ranks' rows over the slowest rank's time
    us_per_row = elapsed_max / (args.steps * step_rows() * world)
    forms_us_per_row = {k: v / (args.steps * step_rows() * world) for k, v in form_us.items()}
    clocks_best = dict(clocks[best_form])
    clocks_best["other_form"] = clocks[[k for k in clocks if k != best_form][0]]
    del forms

    # ---- per-m curves and the GEMV roofline (back-to-back graph-captured calls)
    curves = gemv_curves(rb, flags, hbm_peak)
    curve = curves["router"]
    # Dominant kernel: the fused router kernel (the step's only kernel),
    # averaged over the step's mix of m.  Algorithmic bytes of a window: the
    # weight once, A, and the top-10 indices and values; the logits stay an
    # intermediate (in L2).  Its time: back-to-back graph-captured windows.
    fused_us = sum(curve[str(m)]["router_fused_us_per_window"] for m in WINDOWS) / len(WINDOWS)
    fused_bytes = sum(router_bytes(m) for m in WINDOWS) / len(WINDOWS)
    achieved = fused_bytes / (fused_us * 1e3)
    mean_call_us = sum(curve[str(m)]["us_per_call"] for m in WINDOWS) / len(WINDOWS)
    mean_bytes = sum(gemv_bytes(m, N_ROUTER, K_ROUTER) for m in WINDOWS) / len(WINDOWS)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": recorded_traffic("router_fused"),
                "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                "peak_kind": f"{peak_kind} copy bandwidth",
                "kernel": "router_gemv_topk fused kernel (GEMV + top-10 tail; router, m mix 1..16)",
                "algorithmic_bytes_per_launch": fused_bytes, "us_per_launch": fused_us,
                "gemv_only": {"kernel": "mrgemv_bf16 (router, m mix 1..16)",
                              "achieved": mean_bytes / (mean_call_us * 1e3),
                              "frac": mean_bytes / (mean_call_us * 1e3) / hbm_peak,
                              "algorithmic_bytes_per_launch": mean_bytes, "us_per_launch": mean_call_us,
                              "traffic": recorded_traffic("gemv_router")}}
    # The FFN and sweep weights (8.7 and 31 MB) are large enough to be HBM-bound:
    # their fractions of the measured copy bandwidth, m = 1..8, reported apart.
    roofline["by_shape_m1_to_8"] = {name: {m: curves[name][str(m)]["frac_of_measured_hbm"] for m in (1, 2, 4, 8)}
                                    for name, _, _ in GEMV_SHAPES}
    roofline["by_shape_m1_to_8_of_nominal_8tbs"] = {
        name: {m: curves[name][str(m)]["GBps"] / NOMINAL_HBM_GBS for m in (1, 2, 4, 8)} for name, _, _ in GEMV_SHAPES}

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(rb, args, world, device, fused=True)

    # ---- GEMM sweep (prompt-chunk shapes) and the m-sweep over both paths
    gemm = run_gemm_sweep(args) if not args.skip_gemm else None
    sweep = path_sweep() if not (args.skip_gemm or args.quick) else None

    # ---- CPU oracle baseline (rank 0, N=1 only)
    cpu, cpus = None, None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = cpu_baseline(rb)
        cpus = cpu_baselines()

    if rank == 0:
        line = {
            "metric": "us_per_row", "value": us_per_row, "unit": "us/row", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_max / args.steps / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(),
            "gpu_launches": args.steps * len(WINDOWS) * (1 if best_form == "fused" else 2),
            "forms_us_per_row": forms_us_per_row,
            "device_errors": errs, "clocks": clocks_best, "roofline": roofline,
            "curve": curves,
            "e2e": e2e, "gemm": gemm, "path_sweep": sweep, "cpu_baseline": cpu, "cpu_baselines": cpus,
            "pdl": not args.no_pdl,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


ROUNDS = 5


def graph_of(torch, stream, fn):
    """Capture fn() once into a CUDA graph on `stream` (after one eager run)."""
    with torch.cuda.stream(stream):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    g.replay()
    torch.cuda.synchronize()
    return g


def replay_us(torch, stream, graph, reps):
    """Device time of `reps` back-to-back replays (CUDA events on `stream`), in us."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3


def interleaved(torch, stream, cases, rounds=ROUNDS):
    """Time every case once per round, the cases interleaved, for `rounds` rounds.

    A case is (key, graph, units, reps): `units` calls per replay.  Returns
    {key: {"min": us per unit, "median": us per unit, "samples": [...]}}; min is
    the primary figure, as in the audit's method (min over interleaved rounds)."""
    samples = {key: [] for key, _, _, _ in cases}
    for _ in range(rounds):
        for key, g, units, reps in cases:
            samples[key].append(replay_us(torch, stream, g, reps) / (reps * units))
    return {k: {"min": min(v), "median": statistics.median(v), "samples": v} for k, v in samples.items()}


GEMV_SHAPES = (("router", K_ROUTER, N_ROUTER), ("ffn_k896_n4864", 896, 4864), ("sweep_k2560_n6144", 2560, 6144))


def gemv_curves(rb, flags, hbm_peak):
    """us per call and per row, GB/s and the fraction of the measured HBM copy
    bandwidth for each window size m, on the router, FFN and sweep weights;
    each from graphs of back-to-back calls over distinct weight copies (more
    than 2x the L2), min and median over interleaved rounds.  Also the
    per-row-launch mode (m calls of m = 1, the unbatched baseline) and, on the
    router, the fused and two-launch router windows."""
    import numpy as np
    import synth
    torch, mr = rb.torch, rb.mr
    stream = rb.stream
    cases, meta = [], {}
    keep = []
    for name, k, n in GEMV_SHAPES:
        if name == "router":
            pool, A = rb.W, rb.A
        else:
            wl = synth.WL_GEMV_FFN if k == 896 else synth.WL_SWEEP
            a16 = synth.normal_bits(synth.seed_for(wl, 0), (16, k), "bf16", 1.0)
            w16 = synth.normal_bits(synth.seed_for(wl, 1), (n, k), "bf16", 1.0 / np.sqrt(k))
            w = torch.from_numpy(w16.view(np.int16)).to(rb.device)
            pool = [w.clone() for _ in range(max(4, int(math.ceil(2.2 * rb.l2 / w16.nbytes))))]
            A = torch.from_numpy(a16.view(np.int16)).to(rb.device)
        launches = min(len(pool), 64) if name == "router" else max(len(pool), 16)
        C = torch.empty((16, n), dtype=torch.float32, device=rb.device)
        keep.append((pool, A, C))
        for m in WINDOWS:
            def batched(m=m, pool=pool, A=A, C=C, launches=launches):
                for i in range(launches):
                    mr.mrgemv_bf16(A[:m], pool[i % len(pool)], C[:m], flags=flags)

            def per_row(m=m, pool=pool, A=A, C=C, launches=launches):
                for i in range(max(1, launches // m)):
                    for r in range(m):
                        mr.mrgemv_bf16(A[r:r + 1], pool[i % len(pool)], C[r:r + 1], flags=flags)
            def warm(m=m, pool=pool, A=A, C=C, launches=launches):
                for _ in range(launches):
                    mr.mrgemv_bf16(A[:m], pool[0], C[:m], flags=flags)
            cases.append(((name, m, "batched"), graph_of(torch, stream, batched), launches, 4))
            cases.append(((name, m, "warm"), graph_of(torch, stream, warm), launches, 4))
            cases.append(((name, m, "per_row"), graph_of(torch, stream, per_row), max(1, launches // m), 2))
            meta[(name, m)] = gemv_bytes(m, n, k)
            if name == "router":
                idx = torch.empty((m, TOPK), dtype=torch.int32, device=rb.device)
                val = torch.empty((m, TOPK), dtype=torch.float32, device=rb.device)
                keep.append((idx, val))

                def fused(m=m, idx=idx, val=val, launches=launches):
                    for i in range(launches):
                        mr.router_gemv_topk(A[:m], pool[i % len(pool)], TOPK, idx, val, workspace=rb.ws, flags=flags)

                def two(m=m, idx=idx, val=val, launches=launches):
                    for i in range(launches):
                        mr.mrgemv_bf16(A[:m], pool[i % len(pool)], C[:m], flags=flags)
                        mr.router_topk(C[:m], TOPK, idx, val)
                cases.append(((name, m, "fused"), graph_of(torch, stream, fused), launches, 2))
                cases.append(((name, m, "two_launch"), graph_of(torch, stream, two), launches, 2))
    t = interleaved(torch, stream, cases)
    out = {}
    for name, k, n in GEMV_SHAPES:
        cur = {}
        for m in WINDOWS:
            b = t[(name, m, "batched")]
            nbytes = meta[(name, m)]
            row = {"us_per_call": b["min"], "us_per_call_median": b["median"], "us_per_row": b["min"] / m,
                   "GBps": nbytes / (b["min"] * 1e3), "frac_of_measured_hbm": nbytes / (b["min"] * 1e3) / hbm_peak,
                   "per_row_launch_us_per_row": t[(name, m, "per_row")]["min"] / m,
                   "us_per_call_warm_l2": t[(name, m, "warm")]["min"]}
            if name == "router":
                row["router_fused_us_per_window"] = t[(name, m, "fused")]["min"]
                row["router_two_launch_us_per_window"] = t[(name, m, "two_launch")]["min"]
            cur[str(m)] = row
        cur["batching_speedup_m1_over_m8"] = cur["1"]["us_per_row"] / cur["8"]["us_per_row"]
        out[name] = cur
    out["method"] = (f"min (and median) over {ROUNDS} interleaved rounds of graph-replayed back-to-back calls; "
                     "weights rotated over copies > 2x L2 (us_per_call_warm_l2: the same weight every call)")
    del cases, keep
    return out


def run_e2e(rb, args, world, device, fused=True):
    """K steps through the public API: host A -> device, GEMV, top-10, indices -> host."""
    import numpy as np
    import torch
    mr = rb.mr
    flags = 0 if args.no_pdl else mr.MR_GEMV_PDL
    # The step's rows for every window, stacked (1 + 2 + 4 + 8 + 16 = 31 rows):
    # one host -> device copy of all inputs and one device -> host copy of the
    # results per step, with each window's calls on its slice.
    rows = step_rows()
    offs, o = {}, 0
    for m in WINDOWS:
        offs[m] = o
        o += m
    a_rows = np.concatenate([rb.a16[:m] for m in WINDOWS]).view(np.int16)
    a_host = torch.from_numpy(a_rows).pin_memory()
    # Indices and values of a row side by side in one buffer (the API takes
    # them with a common row stride), so one copy brings both back.
    out_host = torch.empty((rows, 2 * TOPK), dtype=torch.int32).pin_memory()
    a_dev = torch.empty((rows, K_ROUTER), dtype=torch.int16, device=device)
    out_dev = torch.empty((rows, 2 * TOPK), dtype=torch.int32, device=device)
    idx_dev = out_dev[:, :TOPK]
    val_dev = out_dev.view(torch.float32)[:, TOPK:]
    steps = max(1, min(args.steps, 2000))

    # Each window's views of the stacked buffers, made once.
    views = {m: (a_dev[offs[m]:offs[m] + m], idx_dev[offs[m]:offs[m] + m], val_dev[offs[m]:offs[m] + m])
             for m in WINDOWS}

    def one_step():
        a_dev.copy_(a_host, non_blocking=True)
        for m in WINDOWS:
            a_m, idx_m, val_m = views[m]
            mr.router_gemv_topk(a_m, rb._next_w(), TOPK, idx_m, val_m, workspace=rb.ws,
                                flags=flags if fused else flags | mr.MR_ROUTER_TWO_LAUNCH)
        out_host.copy_(out_dev, non_blocking=True)

    with torch.cuda.stream(rb.stream):
        for _ in range(3):
            one_step()
        torch.cuda.synchronize()
        barrier(world)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(rb.stream)
        for _ in range(steps):
            one_step()
        end.record(rb.stream)
    torch.cuda.synchronize()
    us = max_over_ranks(start.elapsed_time(end) * 1e3, world, device)
    # The last step's results, as they reached the host: valid indices, and
    # values in the top-k's order (non-increasing along each row).
    got_idx = out_host[:, :TOPK].numpy()
    got_val = out_host.view(torch.float32)[:, TOPK:].numpy()
    results_ok = bool(((got_idx >= 0) & (got_idx < N_ROUTER)).all() and (np.diff(got_val, axis=1) <= 0).all())
    # The same steps with their public-API calls captured into CUDA graphs,
    # one graph per step on its own slice of the weight pool (weights still
    # from HBM).  The host copies are graph nodes, so every replay moves the
    # bytes: what a caller that replays its window sequence sees, without the
    # per-call Python and launch overhead of the eager loop above.  Every rank
    # takes the same barrier and reductions whether or not its capture worked.
    graphs = []
    try:
        with torch.cuda.stream(rb.stream):
            for _ in range(max(1, rb.pool // len(WINDOWS))):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=rb.stream):
                    one_step()
                graphs.append(g)
            for g in graphs:
                g.replay()
        torch.cuda.synchronize()
    except Exception:
        graphs = []
    barrier(world)
    local = -1.0
    if graphs:
        gs = torch.cuda.Event(enable_timing=True)
        ge = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(rb.stream):
            gs.record(rb.stream)
            for i in range(steps):
                graphs[i % len(graphs)].replay()
            ge.record(rb.stream)
        torch.cuda.synchronize()
        local = gs.elapsed_time(ge) * 1e3
    worst = max_over_ranks(local, world, device)
    ok_all = -max_over_ranks(-local, world, device) >= 0.0
    graph_us = worst if ok_all else None
    del graphs

    # Pipelined: each step's graph also copies the next step's input rows, on
    # a side stream, into the other of two device buffers while its own
    # windows run; the results still come back at the end of every step.  The
    # first step's rows are copied before the timed region, and the last step
    # copies rows that no timed step uses, so the timed region holds exactly
    # one input copy and one result copy per step.
    a_bufs = [a_dev, torch.empty_like(a_dev)]
    side = torch.cuda.Stream(device)

    def piped_step(b):
        cur = torch.cuda.current_stream()
        side.wait_stream(cur)  # the other buffer's last reader (the step before) is done
        with torch.cuda.stream(side):
            a_bufs[1 - b].copy_(a_host, non_blocking=True)
        for m in WINDOWS:
            _, idx_m, val_m = views[m]
            mr.router_gemv_topk(a_bufs[b][offs[m]:offs[m] + m], rb._next_w(), TOPK, idx_m, val_m,
                                workspace=rb.ws, flags=flags if fused else flags | mr.MR_ROUTER_TWO_LAUNCH)
        cur.wait_stream(side)
        out_host.copy_(out_dev, non_blocking=True)

    pgraphs = []
    try:
        with torch.cuda.stream(rb.stream):
            count = max(2, (rb.pool // len(WINDOWS)) // 2 * 2)
            for j in range(count):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=rb.stream):
                    piped_step(j % 2)
                pgraphs.append(g)
            a_bufs[0].copy_(a_host, non_blocking=True)
            for g in pgraphs:
                g.replay()
        torch.cuda.synchronize()
    except Exception:
        pgraphs = []
    barrier(world)
    local = -1.0
    if pgraphs:
        with torch.cuda.stream(rb.stream):
            a_bufs[0].copy_(a_host, non_blocking=True)
        torch.cuda.synchronize()
        gs = torch.cuda.Event(enable_timing=True)
        ge = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(rb.stream):
            gs.record(rb.stream)
            for i in range(steps - steps % 2):
                pgraphs[i % len(pgraphs)].replay()
            ge.record(rb.stream)
        torch.cuda.synchronize()
        local = gs.elapsed_time(ge) * 1e3 / max(1, steps - steps % 2) * steps
    worst = max_over_ranks(local, world, device)
    ok_all = -max_over_ranks(-local, world, device) >= 0.0
    piped_us = worst if ok_all else None
    del pgraphs
    h2d = sum(m * K_ROUTER * 2 for m in WINDOWS)
    d2h = sum(m * TOPK * 8 for m in WINDOWS)
    return {"value": us / (steps * step_rows() * world), "unit": "us/row",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "api": "router_gemv_topk" + ("" if fused else " with MR_ROUTER_TWO_LAUNCH (GEMV kernel + top-k kernel)")
                   + " (verify_weight_streaming_b200), one call per window, pinned host buffers",
            "graph_value": (graph_us / (steps * step_rows() * world)) if graph_us is not None else None,
            "pipelined_graph_value": (piped_us / (steps * step_rows() * world)) if piped_us is not None else None,
            "pipelined_note": "graph per step that also copies the next step's input on a side stream "
                              "(two device input buffers); one input and one result copy per step",
            "results_ok": results_ok,
            "graph_note": "same calls and host copies, captured once into a CUDA graph and replayed"}


def cpu_baseline(rb):
    import oracle
    oracle.default()
    steps, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < 10.0 and steps < 200:
        oracle_router_step(rb.a16, rb.w16)
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": dt * 1e6 / (steps * step_rows()), "unit": "us/row", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{steps} router steps (31 rows each: windows m=1,2,4,8,16, 2560x512, top-10)"}


def cpu_baselines():
    """The oracle (plain C, fp64, every host core) beside each of the other
    workloads, each on a bounded sample (a few seconds of CPU work in all)."""
    import numpy as np
    import oracle
    import synth
    oracle.default()
    cores = oracle.num_threads()

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return (time.perf_counter() - t0) * 1e6

    out = {}
    # FFN GEMV (k = 896, n = 4864), every window size of the workload
    ffn = {}
    for m in (1, 2, 4, 8):
        a, w = synth.gemv_ffn(m)
        us = timed(lambda: oracle.matmul(a, "bf16", w, "bf16"))
        ffn[str(m)] = {"us_per_call": us, "us_per_row": us / m, "GFLOPs": 2.0 * m * 4864 * 896 / (us * 1e3)}
    out["ffn_gemv_k896_n4864"] = {"value": ffn["8"]["us_per_row"], "unit": "us/row", "per_m": ffn,
                                  "cores": cores, "kind": "oracle", "sample": "full calls, m = 1, 2, 4, 8"}
    # narrow N = 96 GEMM: one of the 36 projections at M = 512
    a, w = synth.narrow(512)
    us = timed(lambda: oracle.matmul(a, "f16", w, "f16"))
    out["narrow_gemm_n96"] = {"value": us, "unit": "us/call", "GFLOPs": 2.0 * 512 * 96 * 2560 / (us * 1e3),
                              "cores": cores, "kind": "oracle", "sample": "one 512 x 96 x 2560 call of the 36"}
    # prompt-chunk GEMM: a tail-tile shape, rows sampled
    a, w = synth.chunk(306, 1152)
    us = timed(lambda: oracle.matmul(a[:128], "f16", w, "f16"))
    out["chunk_gemm_306x1152"] = {"value": us * 306 / 128, "unit": "us/call",
                                  "GFLOPs": 2.0 * 128 * 1152 * 2560 / (us * 1e3), "cores": cores,
                                  "kind": "oracle", "sample": "128 of the 306 rows, scaled to the call"}
    # m-sweep weights (k = 2560, n = 6144): the GEMV at m = 1 and 16 rows of the GEMM side
    a = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 0), (16, 2560), "bf16", 1.0)
    w = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 1), (6144, 2560), "bf16", 1.0 / np.sqrt(2560))
    us1 = timed(lambda: oracle.matmul(a[:1], "bf16", w, "bf16"))
    us16 = timed(lambda: oracle.matmul(a, "bf16", w, "bf16"))
    out["sweep_k2560_n6144"] = {"value": us16 / 16, "unit": "us/row", "us_per_row_m1": us1,
                                "GFLOPs": 2.0 * 16 * 6144 * 2560 / (us16 * 1e3), "cores": cores,
                                "kind": "oracle", "sample": "m = 1 and m = 16 calls"}
    return out


GEMM_M = (150, 192, 306, 448, 700, 1300, 1983, 2048)
GEMM_N = (512, 640, 1152, 1664, 4096, 6144)
NARROW_M = (512, 640, 768, 1024, 1983, 2048)


def run_gemm_sweep(args):
    import verify_weight_streaming_b200 as mr
    if mr.gemm_f16_num_tiles() <= 0:
        return {"status": "gemm_f16 not built"}
    return gemm_sweep(quick=args.quick)


def _time_calls(torch, calls, reps=3):
    """Graph-capture `calls` (a list of thunks), replay, return us per call (min of reps)."""
    s = torch.cuda.Stream()
    g = graph_of(torch, s, lambda: [c() for c in calls])
    best = min(replay_us(torch, s, g, 1) / len(calls) for _ in range(reps))
    del g
    return best


def gemm_sweep(quick=False):
    """TFLOP/s of gemm_f16 (auto tile) on the prompt-chunk and narrow shapes.

    Each shape is a graph of back-to-back calls that rotate over weight copies
    (and A copies) whose total exceeds twice the L2, so operands come from HBM
    as they would for a chunk's successive projections.  Every shape is timed
    once per round, shapes interleaved, over ROUNDS rounds: min and median."""
    import numpy as np
    import torch
    import synth
    import verify_weight_streaming_b200 as mr
    hbm, tf_burst, tf_sus, kind = load_peaks()
    props = torch.cuda.get_device_properties(0)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    K = 2560
    stream = torch.cuda.Stream()
    ms = GEMM_M if not quick else (306, 2048)
    ns = GEMM_N if not quick else (512, 6144)
    a_all = torch.from_numpy(synth.chunk(max(ms), 16)[0].view(np.int16)).cuda().view(torch.float16)
    w_all = torch.from_numpy(synth.chunk(16, max(ns))[1].view(np.int16)).cuda().view(torch.float16)
    cases, keep, flops = [], [], {}
    for N in ns:
        for M in ms:
            per = (M + N) * K * 2
            copies = int(min(48, max(2, np.ceil(2.2 * l2 / per))))
            As = [a_all[:M].clone() for _ in range(copies)]
            Ws = [w_all[:N].clone() for _ in range(copies)]
            C = torch.empty((M, N), dtype=torch.float16, device="cuda")
            keep.append((As, Ws, C))

            def calls(As=As, Ws=Ws, C=C):
                for A, W in zip(As, Ws):
                    mr.gemm_f16(A, W, C)
            cases.append((("chunk", f"{M}x{N}"), graph_of(torch, stream, calls), copies, 1))
            flops[("chunk", f"{M}x{N}")] = 2.0 * M * N * K
    # narrow: one A per M shared by 36 different W[96, 2560]
    w96 = [torch.from_numpy(synth.narrow(1, w_index=i)[1].view(np.int16)).cuda().view(torch.float16)
           for i in range(36)]
    for M in (NARROW_M if not quick else (2048,)):
        a16 = torch.from_numpy(synth.narrow(M)[0].view(np.int16)).cuda().view(torch.float16)
        C = torch.empty((M, 96), dtype=torch.float16, device="cuda")
        Cs = [torch.empty((M, 96), dtype=torch.float16, device="cuda") for _ in range(36)]
        keep.append((a16, C, Cs))

        def singles(a16=a16, C=C):
            for W in w96:
                mr.gemm_f16(a16, W, C)

        def grouped(a16=a16, Cs=Cs):
            for _ in range(4):
                mr.gemm_f16_grouped(a16, w96, Cs)
        cases.append((("narrow", M), graph_of(torch, stream, singles), 36, 1))
        cases.append((("narrow_grouped", M), graph_of(torch, stream, grouped), 4, 1))
    # Tile-order study (the analogue of the audit's SLC swizzle): same bits,
    # timed for several column-band widths (operands warm in L2).
    same_bits = {}
    for (M, N) in ((2048, 6144), (1983, 4096), (448, 6144)):
        A, W = a_all[:M], w_all[:N]
        ref = None
        for raster in (0, 2, 4, 8):
            C = torch.empty((M, N), dtype=torch.float16, device="cuda")
            keep.append(C)

            def calls(A=A, W=W, C=C, r=raster):
                for _ in range(8):
                    mr.gemm_f16(A, W, C, raster=r)
            cases.append((("raster", f"{M}x{N}", raster), graph_of(torch, stream, calls), 8, 1))
            same_bits[(f"{M}x{N}", raster)] = True if ref is None else bool(
                torch.equal(C.view(torch.int16), ref.view(torch.int16)))
            ref = C if ref is None else ref
    t = interleaved(torch, stream, cases)
    out = {"chunk": {}, "narrow": {}, "raster_study": {}}
    for N in ns:
        for M in ms:
            key = ("chunk", f"{M}x{N}")
            out["chunk"][f"{M}x{N}"] = {"us": t[key]["min"], "us_median": t[key]["median"],
                                        "TFLOPs": flops[key] / (t[key]["min"] * 1e-6) / 1e12,
                                        "tile": mr.gemm_f16_tile_name(mr.gemm_f16_select_tile(M, N, K))}
    for M in (NARROW_M if not quick else (2048,)):
        us, ug = t[("narrow", M)]["min"], t[("narrow_grouped", M)]["min"]
        out["narrow"][str(M)] = {"us_per_call": us, "us_per_call_median": t[("narrow", M)]["median"],
                                 "us_per_36_calls": 36 * us, "TFLOPs": 2.0 * M * 96 * K / (us * 1e-6) / 1e12,
                                 "tile": mr.gemm_f16_tile_name(mr.gemm_f16_select_tile(M, 96, K)),
                                 "grouped_us_for_36": ug, "grouped_us_for_36_median": t[("narrow_grouped", M)]["median"],
                                 "grouped_TFLOPs": 36 * 2.0 * M * 96 * K / (ug * 1e-6) / 1e12,
                                 "grouped_tile": mr.gemm_f16_tile_name(mr.gemm_f16_grouped_select_tile(M, 96, K, 36))}
    for (M, N) in ((2048, 6144), (1983, 4096), (448, 6144)):
        out["raster_study"][f"{M}x{N}"] = {
            str(r): {"us": t[("raster", f"{M}x{N}", r)]["min"],
                     "TFLOPs": 2.0 * M * N * K / (t[("raster", f"{M}x{N}", r)]["min"] * 1e-6) / 1e12,
                     "same_bits": same_bits[(f"{M}x{N}", r)]} for r in (0, 2, 4, 8)}
    big = [v["TFLOPs"] for k, v in out["chunk"].items() if int(k.split("x")[0]) >= 1024]
    big_n = [v["TFLOPs"] for k, v in out["chunk"].items()
             if int(k.split("x")[0]) >= 1024 and int(k.split("x")[1]) >= 4096]
    out["summary"] = {"tflops_M_ge_1024_mean": float(np.mean(big)) if big else None,
                      "tflops_M_ge_1024_max": float(np.max(big)) if big else None,
                      "tflops_M_ge_1024_N_ge_4096_mean": float(np.mean(big_n)) if big_n else None,
                      "peak_bf16_tflops": tf_burst, "peak_bf16_tflops_sustained": tf_sus, "peak_kind": kind,
                      "frac_of_peak_mean": (float(np.mean(big)) / tf_burst) if big else None,
                      "method": f"min (and median) over {ROUNDS} interleaved rounds; operands rotated over "
                                "copies > 2x L2 (raster study: warm)"}
    del cases, keep
    return out


def selector_study():
    """Every tile of gemm_f16 timed on every prompt-chunk shape, against the
    tile the selector picks: regret = t(selected) / t(best) - 1.  Timed like
    gemm_sweep (graph replays over operand copies larger than twice the L2).
    All tiles give the same bits, so this only measures the selection rule."""
    import numpy as np
    import torch
    import synth
    import verify_weight_streaming_b200 as mr
    props = torch.cuda.get_device_properties(0)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    K = 2560
    a_all = torch.from_numpy(synth.chunk(max(GEMM_M), 16)[0].view(np.int16)).cuda().view(torch.float16)
    w_all = torch.from_numpy(synth.chunk(16, max(GEMM_N))[1].view(np.int16)).cuda().view(torch.float16)
    names = [mr.gemm_f16_tile_name(t) for t in range(mr.gemm_f16_num_tiles())]
    shapes, regrets = {}, []
    for N in GEMM_N:
        for M in GEMM_M:
            per = (M + N) * K * 2
            copies = int(min(48, max(2, np.ceil(2.2 * l2 / per))))
            As = [a_all[:M].clone() for _ in range(copies)]
            Ws = [w_all[:N].clone() for _ in range(copies)]
            C = torch.empty((M, N), dtype=torch.float16, device="cuda")
            times = {}
            for t, name in enumerate(names):
                calls = [(lambda A=As[i], W=Ws[i], t=t: mr.gemm_f16(A, W, C, tile_id=t)) for i in range(copies)]
                times[name] = _time_calls(torch, calls)
            sel = names[mr.gemm_f16_select_tile(M, N, K)]
            best = min(times, key=times.get)
            regret = times[sel] / times[best] - 1.0
            regrets.append(regret)
            shapes[f"{M}x{N}"] = {"us": times, "selected": sel, "best": best, "regret": regret}
            del As, Ws, C
    return {"K": K, "shapes": shapes,
            "summary": {"mean_regret": float(np.mean(regrets)), "max_regret": float(np.max(regrets)),
                        "best_picked": int(sum(1 for r in regrets if r <= 1e-9)), "shapes": len(regrets)}}


SWEEP_M = (1, 2, 4, 8, 16, 32, 64, 128, 256, 306, 512, 1024, 1983, 2048)


def path_sweep():
    """The m-sweep over both paths on the FFN (k=896, n=4864) and the
    (k=2560, n=6144) weights: us_per_row of the multi-row GEMV (m > 16 runs as
    16-row groups, each re-reading the weight) and of the tcgen05 GEMM (bf16
    in, fp32 out, auto tile), and the smallest m at which the GEMM is faster.
    Weights rotate over copies larger than 2x L2; min and median over
    interleaved rounds."""
    import numpy as np
    import torch
    import synth
    import verify_weight_streaming_b200 as mr
    props = torch.cuda.get_device_properties(0)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    stream = torch.cuda.Stream()
    cases, keep = [], []
    for name, k, n, wl in (("k896_n4864", 896, 4864, synth.WL_GEMV_FFN),
                           ("k2560_n6144", 2560, 6144, synth.WL_SWEEP)):
        a16 = synth.normal_bits(synth.seed_for(wl, 0), (max(SWEEP_M), k), "bf16", 1.0)
        w16 = synth.normal_bits(synth.seed_for(wl, 1), (n, k), "bf16", 1.0 / np.sqrt(k))
        A = torch.from_numpy(a16.view(np.int16)).cuda()
        w = torch.from_numpy(w16.view(np.int16)).cuda()
        copies = max(3, int(np.ceil(2.2 * l2 / w16.nbytes)))
        Ws = [w.clone() for _ in range(copies)]
        Ab = A.view(torch.bfloat16)
        Wb = [x.view(torch.bfloat16) for x in Ws]
        keep.append((A, Ws))
        for m in SWEEP_M:
            C = torch.empty((m, n), dtype=torch.float32, device="cuda")
            keep.append(C)
            groups = [(r0, min(16, m - r0)) for r0 in range(0, m, 16)]

            def gemv_calls(C=C, groups=groups):
                for W in Ws:
                    for r0, rr in groups:
                        mr.mrgemv_bf16(A[r0:r0 + rr], W, C[r0:r0 + rr], flags=mr.MR_GEMV_PDL)

            def gemm_calls(C=C, m=m):
                for W in Wb:
                    mr.gemm_f16(Ab[:m], W, C)
            cases.append(((name, m, "gemv"), graph_of(torch, stream, gemv_calls), copies, 1))
            cases.append(((name, m, "gemm"), graph_of(torch, stream, gemm_calls), copies, 1))
    t = interleaved(torch, stream, cases)
    res = {}
    for name, k, n in (("k896_n4864", 896, 4864), ("k2560_n6144", 2560, 6144)):
        curve, cross = {}, None
        for m in SWEEP_M:
            t_gemv, t_gemm = t[(name, m, "gemv")]["min"], t[(name, m, "gemm")]["min"]
            curve[str(m)] = {"gemv_us_per_row": t_gemv / m, "gemm_us_per_row": t_gemm / m,
                             "gemv_us": t_gemv, "gemm_us": t_gemm,
                             "gemv_us_median": t[(name, m, "gemv")]["median"],
                             "gemm_us_median": t[(name, m, "gemm")]["median"],
                             "gemm_TFLOPs": 2.0 * m * n * k / (t_gemm * 1e-6) / 1e12,
                             "gemm_tile": mr.gemm_f16_tile_name(mr.gemm_f16_select_tile(m, n, k))}
            if cross is None and t_gemm <= t_gemv:
                cross = m
        res[name] = {"curve": curve, "crossover_m": cross,
                     "note": "GEMV for m > 16 is ceil(m/16) calls of up to 16 rows; GEMM is one call"}
    del cases, keep
    return res


def gemm_profile_case():
    """A few GEMM launches on a 2048 x 6144 x 2560 chunk shape (for ncu)."""
    import numpy as np
    import torch
    import synth
    import verify_weight_streaming_b200 as mr
    a, w = synth.chunk(2048, 6144)
    A = torch.from_numpy(a.view(np.int16)).cuda().view(torch.float16)
    W = torch.from_numpy(w.view(np.int16)).cuda().view(torch.float16)
    C = torch.empty((2048, 6144), dtype=torch.float16, device="cuda")
    for _ in range(3):
        mr.gemm_f16(A, W, C)
    a, w = synth.narrow(2048)
    A = torch.from_numpy(a.view(np.int16)).cuda().view(torch.float16)
    W = torch.from_numpy(w.view(np.int16)).cuda().view(torch.float16)
    C = torch.empty((2048, 96), dtype=torch.float16, device="cuda")
    for _ in range(3):
        mr.gemm_f16(A, W, C)


# ------------------------------------------------------------------- profiling

def profile_case(case: str):
    """A handful of launches on a small case, for ncu captures (no timing)."""
    import numpy as np
    import torch
    import synth
    import verify_weight_streaming_b200 as mr
    torch.cuda.set_device(0)
    if case == "gemv":
        a16, w16 = synth.router(16)
        # a pool > L2 so the captured launch reads its weight from DRAM
        pool = [torch.from_numpy(w16.view(np.int16)).cuda() for _ in range(110)]
        A = torch.from_numpy(a16.view(np.int16)).cuda()
        for m in WINDOWS:
            C = torch.empty((m, N_ROUTER), dtype=torch.float32, device="cuda")
            for i in range(4):
                mr.mrgemv_bf16(A[:m], pool[(7 * i + m) % len(pool)], C)
    elif case in ("gemv_ffn", "gemv_sweep"):
        k, n, wl, m = (896, 4864, synth.WL_GEMV_FFN, 16) if case == "gemv_ffn" else (2560, 6144, synth.WL_SWEEP, 8)
        a16 = synth.normal_bits(synth.seed_for(wl, 0), (16, k), "bf16", 1.0)
        w16 = synth.normal_bits(synth.seed_for(wl, 1), (n, k), "bf16", 1.0 / np.sqrt(k))
        W = [torch.from_numpy(w16.view(np.int16)).cuda() for _ in range(8)]
        A = torch.from_numpy(a16.view(np.int16)).cuda()
        C = torch.empty((m, n), dtype=torch.float32, device="cuda")
        for i in range(3):
            mr.mrgemv_bf16(A[:m], W[i], C)
    elif case == "fused":
        # the fused router kernel alone, 4 launches per m, weight from DRAM
        a16, w16 = synth.router(16)
        pool = [torch.from_numpy(w16.view(np.int16)).cuda() for _ in range(110)]
        A = torch.from_numpy(a16.view(np.int16)).cuda()
        ws = torch.zeros(mr.router_gemv_topk_workspace_bytes(16, N_ROUTER, False) // 4 + 1,
                         dtype=torch.int32, device="cuda")
        for m in WINDOWS:
            idx = torch.empty((m, TOPK), dtype=torch.int32, device="cuda")
            val = torch.empty((m, TOPK), dtype=torch.float32, device="cuda")
            for i in range(4):
                mr.router_gemv_topk(A[:m], pool[(7 * i + m) % len(pool)], TOPK, idx, val, workspace=ws)
    elif case == "router_fused":
        a16, w16 = synth.router(16)
        pool = [torch.from_numpy(w16.view(np.int16)).cuda() for _ in range(110)]
        A = torch.from_numpy(a16.view(np.int16)).cuda()
        ws = torch.zeros(mr.router_gemv_topk_workspace_bytes(16, N_ROUTER, False) // 4 + 1,
                         dtype=torch.int32, device="cuda")
        for m in (1, 16):
            C = torch.empty((m, N_ROUTER), dtype=torch.float32, device="cuda")
            idx = torch.empty((m, TOPK), dtype=torch.int32, device="cuda")
            val = torch.empty((m, TOPK), dtype=torch.float32, device="cuda")
            for i in range(3):
                mr.mrgemv_bf16(A[:m], pool[(3 * i + m) % len(pool)], C)
                mr.router_topk(C, TOPK, idx, val)
            for i in range(3):
                mr.router_gemv_topk(A[:m], pool[(5 * i + m + 40) % len(pool)], TOPK, idx, val, workspace=ws)
    elif case == "topk":
        x = torch.randn(16, 512, device="cuda")
        idx = torch.empty((16, TOPK), dtype=torch.int32, device="cuda")
        for _ in range(4):
            mr.router_topk(x, TOPK, idx)
    elif case == "gemm":
        gemm_profile_case()
    elif case == "gemm_1983x1152":
        # a one-wave chunk shape on the auto tile (the 256 x 128 pair)
        a, w = synth.chunk(1983, 1152)
        A = torch.from_numpy(a.view(np.int16)).cuda().view(torch.float16)
        W = torch.from_numpy(w.view(np.int16)).cuda().view(torch.float16)
        C = torch.empty((1983, 1152), dtype=torch.float16, device="cuda")
        for _ in range(3):
            mr.gemm_f16(A, W, C)
    torch.cuda.synchronize()
    assert mr.mr_poll_errors() == 0
    print(json.dumps({"profile_case": case, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="mrgemm", choices=["mrgemm", "reference"])
    ap.add_argument("--no-pdl", action="store_true")
    ap.add_argument("--skip-gemm", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--quick", action="store_true")
    ap.add_argument("--profile-case", default=None)
    ap.add_argument("--selector-study", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_env()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.selector_study:
        print(json.dumps(selector_study()), flush=True)
        return
    if args.impl == "reference":
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    run_gpu(args, world, rank, local)


if __name__ == "__main__":
    main()
