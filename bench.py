"""Benchmark: one exact Lloyd iteration (assignment + sort-inverse update) per step.

Workload (the one the headline metric is quoted on): B=32 independent problems, N=65536 points
each, d=128, K=1024 centroids, fp16 points, fp32 centroids; 1024-component Gaussian mixture per
batch (means N(0,1)^128, sigma=0.3), init = K seeded-random points. Inputs (X = 537 MB) are
larger than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --out-of-core {batched_assign_bound,single_N33M_K16384} --steps 5
  python bench.py --workload {tiny_exact,rows_weighted_1d,large_k_assign,contention_update,emeans,
                              codebook1d}

A step on the GPU = km_assign (tensor-core FlashAssign; the labels, which is all a Lloyd
iteration needs: the per-point distance and the inertia are optional outputs) +
km_update_partial (histogram, scan, scatter, segmented reduce) + km_finalize (the division, with
the rounded centroids and their norms for the next assignment written by the same kernel):
exactly one iteration of km_fit's loop without the objective. The
assignment with the inertia requested is timed separately and reported as
"assign_with_inertia_ms". Multi-GPU: one process per GPU (torchrun),
each rank runs its own B=32 workload (independent problems, no data-path collective, weak
scaling); the step time is the max over ranks.

`--impl reference` times the fp64 CPU oracle on this host (a bounded sample of the same
workload, scaled to the full iteration) and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Lloyd iter/s & assign pt·K/s (B=32,N=65536,K=1024,d=128); % roofline"
B, N, K, D = 32, 65536, 1024, 128
WORKLOAD = "batched_assign_bound: B=32 N=65536 d=128 K=1024 fp16, per-batch 1024-comp GMM sigma=0.3"
ASSIGN_FLOP = 2.0 * B * N * K * D                       # <x,c> contraction per iteration
# algorithmic bytes of the update: X gathered once + ids read twice + perm written and read
UPDATE_BYTES = B * N * D * 2 + 4 * B * N * 4 + B * K * D * 4 * 2
ASSIGN_BYTES = B * N * D * 2 + B * K * D * 2 + B * N * 4
LAUNCHES_PER_STEP = 7   # caug, assign_tc, hist, scan, scatter, segreduce, finalize (+ rounding)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["bf16_tflops"]), float(j["hbm_gbs"]), "measured"
    return 1590.0, 6650.0, "fallback"


def _kernel_source_hash():
    h = hashlib.sha256()
    for f in ("km_assign_tc.cuh", "km_common.cuh"):
        with open(os.path.join(ROOT, "exact_lloyd_means_assign_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _profile_traffic():
    """DRAM bytes per assign launch from the committed ncu summary, if it matches this source."""
    p = os.path.join(ROOT, "profiles", "assign_tc_batched_assign_bound.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    s = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    if not m or not s or s.group(1) != _kernel_source_hash():
        return None
    return float(m.group(1))


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        sm = sorted(r[0] for r in rows)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_gpu(args):
    import exact_lloyd_means_assign_b200 as km
    import synth

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    # each rank owns its own B=32 problems (independent batches)
    d = synth.make_workload(3, device=dev, seed=1234 + 3 + 1000 * rank)
    X, C = d["X"], d["C0"]
    ws_a = km.workspace(km.KM_OP_ASSIGN, B, N, K, D, X.dtype, dev)
    ws_u = km.workspace(km.KM_OP_UPDATE, B, N, K, D, X.dtype, dev)
    ids = torch.empty((B, N), dtype=torch.int32, device=dev)
    counts = torch.empty((B, K), dtype=torch.int32, device=dev)
    sums = torch.empty((B, K, D), dtype=torch.float32, device=dev)
    inertia = torch.empty((B,), dtype=torch.float64, device=dev)
    Cx, cn = km.km_prep(C, X.dtype)
    stream = torch.cuda.current_stream()

    def update():
        km.km_update_partial(X, ids, K, sums=sums, counts=counts, ws=ws_u, stream=stream)
        km.km_finalize(sums, counts, C, C_new=C, Cx=Cx, cn=cn, stream=stream)

    def step():
        km.km_assign(X, Cx, cn, ids=ids, ws=ws_a, stream=stream)
        update()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as cs:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            e = ev[i]
            e[0].record(stream)
            km.km_assign(X, Cx, cn, ids=ids, ws=ws_a, stream=stream)
            e[1].record(stream)
            update()
            e[2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    total_ms = t0.elapsed_time(t1)
    assign_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    update_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    # the assignment with the objective requested (per-batch inertia), outside the timed steps
    n_in = max(3, min(50, args.steps // 10))
    for _ in range(3):
        km.km_assign(X, Cx, cn, ids=ids, inertia=inertia, ws=ws_a, stream=stream)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(n_in):
        km.km_assign(X, Cx, cn, ids=ids, inertia=inertia, ws=ws_a, stream=stream)
    a1.record(stream)
    torch.cuda.synchronize()
    assign_inertia_ms = a0.elapsed_time(a1) / n_in
    vals = torch.tensor([total_ms, assign_ms, update_ms, assign_inertia_ms], dtype=torch.float64,
                        device=dev)
    if pg:
        pg.all_reduce(vals, op=pg.ReduceOp.MAX)
    total_ms, assign_ms, update_ms, assign_inertia_ms = vals.tolist()
    ms_per_step = total_ms / args.steps
    err = km.km_device_error()

    # end to end through the public host-buffer entry point: H2D of X and C, one iteration,
    # D2H of the new centroids and the inertia, synchronised, every step
    Xh = X.cpu().pin_memory()
    Ch = d["C0"].cpu().pin_memory()
    inh = torch.empty((1, B), dtype=torch.float64).pin_memory()
    ws_h = km.workspace(km.KM_OP_FIT_HOST, B, N, K, D, X.dtype, dev, False, 1)
    e2e_steps = max(3, min(20, args.steps // 25))
    km.km_fit_host(Xh, Ch, 1, inertia_host=inh, ws=ws_h, device=dev)
    if pg:
        pg.barrier()
    t = time.perf_counter()
    for _ in range(e2e_steps):
        km.km_fit_host(Xh, Ch, 1, inertia_host=inh, ws=ws_h, device=dev)
    e2e_s = torch.tensor([(time.perf_counter() - t) / e2e_steps], dtype=torch.float64, device=dev)
    if pg:
        pg.all_reduce(e2e_s, op=pg.ReduceOp.MAX)
    e2e_s = float(e2e_s.item())

    clocks = cs.summary()
    if rank == 0:
        peak_tf, peak_bw, peak_kind = _peaks()
        achieved_tf = ASSIGN_FLOP / (assign_ms * 1e-3) / 1e12
        upd_gbs = UPDATE_BYTES / (update_ms * 1e-3) / 1e9
        traffic = _profile_traffic()
        line = {
            "metric": METRIC,
            "value": ws * 1e3 / ms_per_step,
            "unit": "iter/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "N": N, "K": K, "d": D, "iterations_per_step": 1,
                       "init": "K seeded-random points per batch", "l2": "inputs larger than L2 (X = 537 MB)",
                       "parallelism": f"batch-sharded x{ws} (independent problems, no collective)"},
            "assign_pt_k_per_s": ws * B * N * K / (assign_ms * 1e-3),
            "assign_ms": assign_ms,
            "update_ms": update_ms,
            "assign_with_inertia_ms": assign_inertia_ms,
            "roofline": {"bound": "tensor", "kernel": "assign_tc_kernel (+ caug_kernel, the centroid side of the norm step)",
                         "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": achieved_tf / peak_tf, "traffic": traffic,
                         "peak_source": f"{peak_kind} bf16 dense (fp16 nominal ratio 1.0)"},
            "update_roofline": {"bound": "hbm", "achieved": upd_gbs, "peak": peak_bw, "unit": "GB/s",
                                "frac": upd_gbs / peak_bw, "algorithmic_bytes": UPDATE_BYTES,
                                "peak_source": peak_kind},
            "e2e": {"value": ws / e2e_s, "unit": "iter/s",
                    "h2d_bytes_per_step": B * N * D * 2 + B * K * D * 4,
                    "d2h_bytes_per_step": B * K * D * 4 + B * 8},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clocks,
            "device_error": err,
        }
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(X, d["C0"], budget_s=args.cpu_budget)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def cpu_baseline(X, C, budget_s=15.0):
    """The fp64 oracle on a bounded sample of the workload, scaled to one full iteration.

    The sample is the first points of batch 0, then of batch 1, ... (assign + update on each
    batch's own centroids) until about ``budget_s`` seconds of CPU work have been measured.
    """
    import oracle
    Cb = oracle.round_to_dtype(C[0:1].cpu(), X.dtype)
    t = time.perf_counter()
    oracle.assign(oracle.as_f64(X[0:1, :1024].cpu()), Cb)
    per_pt = (time.perf_counter() - t) / 1024
    target = int(min(B * N, max(1024, budget_s * 0.9 / max(per_pt, 1e-9))))
    done, measured, nb = 0, 0.0, 0
    for b in range(B):
        if done >= target:
            break
        n = int(min(N, max(1024, target - done)))
        Xb = oracle.as_f64(X[b:b + 1, :n].cpu())
        Cb = oracle.round_to_dtype(C[b:b + 1].cpu(), X.dtype)
        t = time.perf_counter()
        ids, _, _, _ = oracle.assign(Xb, Cb)
        oracle.update(Xb, ids, Cb)
        measured += time.perf_counter() - t
        done += n
        nb += 1
    full = measured * (B * N) / done
    return {"value": 1.0 / full, "unit": "iter/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{done} points from the first {nb} batch(es) (assign + update, fp64), "
                      f"{measured:.1f} s measured, scaled by {B * N / done:.2f} to one full iteration",
            "seconds_measured": measured}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    import oracle
    import synth
    d = synth.make_workload(3, B=1, N=N, device="cpu")
    X, C = d["X"], d["C0"]
    # a step = one bounded sample (assign + update) scaled to the full iteration
    per_step_budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(X, C, budget_s=per_step_budget)
    vals = []
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(X, C, budget_s=per_step_budget)
        vals.append(1.0 / last["value"])
    s_per_iter = sum(vals) / len(vals)
    line = {
        "metric": METRIC, "impl": "reference", "value": 1.0 / s_per_iter, "unit": "iter/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_per_iter * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "N": N, "K": K, "d": D, "iterations_per_step": 1},
        "cpu_baseline": {"value": 1.0 / s_per_iter, "unit": "iter/s", "cores": last["cores"],
                         "kind": "oracle", "sample": last["sample"]},
        "e2e": {"value": 1.0 / s_per_iter, "unit": "iter/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _timed(fn, steps, stream):
    """Mean device ms of fn() over ``steps`` calls (CUDA events on ``stream``)."""
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        fn()
    t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def _steps_for(fn, steps, stream, min_s=0.5):
    """At least ``steps``, and enough for ``min_s`` seconds so that the clock sampler (100 ms
    period) sees the timed region."""
    t = _timed(fn, 2, stream)
    return max(steps, int(min_s * 1e3 / max(t, 1e-3)) + 1)


def run_workload(args):
    """The other synthetic workloads of the measurement table, one JSON line each, 1 GPU:
    tiny_exact (latency, fp32 exact path, eager and CUDA-graph replay of a 20-iteration fit),
    rows_weighted_1d (the fused per-row 1-D fit, K=16 and K=8, ALU roofline),
    large_k_assign and contention_update (one Lloyd iteration per step: tensor-core roofline
    for the assignment, HBM roofline for the sort-inverse update)."""
    import exact_lloyd_means_assign_b200 as km
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    wl = synth.WORKLOADS[{w.name: i for i, w in synth.WORKLOADS.items()}[args.workload]]
    peak_tf, peak_bw, peak_kind = _peaks()
    base = {"n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "none", "vs_baseline": None, "data": "synthetic",
            "dtype": {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[wl.dtype]}
    lines = []
    if wl.name == "tiny_exact":
        d = synth.make_workload(wl.idx, device=dev)
        X, C0 = d["X"], d["C0"]
        Bw, Nw, Dw = X.shape
        Kw, iters = C0.shape[1], d["iters"]
        ws = km.workspace(km.KM_OP_FIT, Bw, Nw, Kw, Dw, X.dtype, dev)
        C = C0.clone()

        def fit():   # on the current stream: the capture stream while the graph is recorded
            C.copy_(C0)
            km.km_fit(X, C, iters, ws=ws)

        for _ in range(args.warmup):
            fit()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fit()
        steps = _steps_for(g.replay, args.steps, stream)
        with ClockSampler(0) as clk:
            eager = _timed(fit, steps, stream)
            graph = _timed(g.replay, steps, stream)
        lines.append(dict(base, metric="exact fp32 Lloyd us/iteration (CUDA-core path)",
                          value=graph * 1e3 / iters, unit="us/iter", higher_is_better=False,
                          ms_per_step=graph, steps=steps,
                          eager_us_per_iter=eager * 1e3 / iters,
                          config={"workload": wl.name, "B": Bw, "N": Nw, "K": Kw, "d": Dw,
                                  "iterations_per_step": iters, "launch": "CUDA graph of one km_fit call"},
                          roofline={"bound": "latency", "note": "4.2 MFLOP per iteration; launch-bound"},
                          clocks=clk.summary()))
    elif wl.name == "rows_weighted_1d":
        for Kw in wl.K:
            d = synth.make_workload(wl.idx, device=dev, K=Kw)
            X, w = d["X"], d["w"]
            Bw, Nw = X.shape[0], X.shape[1]
            iters = d["iters"]
            C = torch.empty((Bw, Kw, 1), dtype=torch.float32, device=dev)

            def fit():
                km.km_init_grid1d(X, Kw, C=C, stream=stream)
                km.km_fit(X, C, iters, w=w, stream=stream)

            for _ in range(args.warmup):
                fit()
            steps = _steps_for(fit, args.steps, stream)
            with ClockSampler(0) as clk:
                ms = _timed(fit, steps, stream)
            clocks = clk.summary()
            # peak: 128 fp32 lanes per SM per clock x SMs x the median SM clock under load
            mhz = clocks.get("sm_mhz") or 1965.0
            alu_peak = 128 * torch.cuda.get_device_properties(dev).multi_processor_count * mhz * 1e6 / 1e12
            ops = 3.0 * Bw * Nw * Kw * iters   # brute-force equivalent: sub, mul, min per pair
            lines.append(dict(base, metric="weighted 1-D per-row fit iter/s (all rows)",
                              value=iters * 1e3 / ms, unit="iter/s", ms_per_step=ms, steps=steps,
                              config={"workload": wl.name, "B": Bw, "N": Nw, "K": Kw, "d": 1,
                                      "iterations_per_step": iters, "weighted": True, "init": "grid"},
                              roofline={"bound": "alu", "achieved": ops / (ms * 1e-3) / 1e12,
                                        "peak": alu_peak, "unit": "Tops/s",
                                        "frac": ops / (ms * 1e-3) / 1e12 / alu_peak,
                                        "note": "achieved counts 3 ops per (point, centroid) pair "
                                                "(brute force); the kernel does fewer (sorted "
                                                "centroids), so frac may exceed 1",
                                        "peak_source": "128 fp32 lanes/SM/clk x SMs x median SM clock"},
                              hbm_bytes_per_fit=Bw * Nw * (X.element_size() + 4),
                              clocks=clocks))
    else:
        d = synth.make_workload(wl.idx, device=dev)
        X, C = d["X"], d["C0"]
        Bw, Nw, Dw = X.shape
        Kw = C.shape[1]
        ws_a = km.workspace(km.KM_OP_ASSIGN, Bw, Nw, Kw, Dw, X.dtype, dev)
        ws_u = km.workspace(km.KM_OP_UPDATE, Bw, Nw, Kw, Dw, X.dtype, dev)
        ids = torch.empty((Bw, Nw), dtype=torch.int32, device=dev)
        counts = torch.empty((Bw, Kw), dtype=torch.int32, device=dev)
        sums = torch.empty((Bw, Kw, Dw), dtype=torch.float32, device=dev)
        Cx, cn = km.km_prep(C, X.dtype)

        def assign():
            km.km_assign(X, Cx, cn, ids=ids, ws=ws_a, stream=stream)

        def update():
            km.km_update_partial(X, ids, Kw, sums=sums, counts=counts, ws=ws_u, stream=stream)
            km.km_finalize(sums, counts, C, C_new=C, Cx=Cx, cn=cn, stream=stream)

        for _ in range(args.warmup):
            assign()
            update()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        with ClockSampler(0) as clk:
            for e in ev:
                e[0].record(stream)
                assign()
                e[1].record(stream)
                update()
                e[2].record(stream)
            torch.cuda.synchronize()
        a_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
        u_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
        flop = 2.0 * Bw * Nw * Kw * Dw
        ubytes = Bw * Nw * Dw * X.element_size() + 4 * Bw * Nw * 4 + Bw * Kw * Dw * 4 * 2
        line = dict(base, metric="Lloyd iter/s & assign pt·K/s; % roofline", value=1e3 / (a_ms + u_ms),
                    unit="iter/s", ms_per_step=a_ms + u_ms, assign_ms=a_ms, update_ms=u_ms,
                    assign_pt_k_per_s=Bw * Nw * Kw / (a_ms * 1e-3),
                    config={"workload": wl.name, "B": Bw, "N": Nw, "K": Kw, "d": Dw,
                            "iterations_per_step": 1, "l2": "inputs larger than L2"},
                    roofline={"bound": "tensor", "kernel": "assign_tc_kernel",
                              "achieved": flop / (a_ms * 1e-3) / 1e12, "peak": peak_tf,
                              "unit": "TFLOP/s", "frac": flop / (a_ms * 1e-3) / 1e12 / peak_tf,
                              "traffic": None, "peak_source": f"{peak_kind} bf16 dense"},
                    update_roofline={"bound": "hbm", "achieved": ubytes / (u_ms * 1e-3) / 1e9,
                                     "peak": peak_bw, "unit": "GB/s",
                                     "frac": ubytes / (u_ms * 1e-3) / 1e9 / peak_bw,
                                     "algorithmic_bytes": ubytes, "peak_source": peak_kind},
                    gpu_launches=LAUNCHES_PER_STEP * args.steps, clocks=clk.summary(),
                    device_error=km.km_device_error())
        lines.append(line)
    for l in lines:
        print(json.dumps(l), flush=True)


def run_emeans(args):
    """e-means against Lloyd on one large problem (the page's heavy setting is 10M points with
    K = 65536; here B=1, N=2^22, K=16384, d=128, fp16, the same kind of mixture): the time of a
    2-epoch e-means run (mini-batches of --emeans-batch points, by default four full waves of
    256-point tiles over 74 SM pairs; alpha0 = 0.3, cosine decay, splitting of
    dead clusters between epochs) next to the time of one exact Lloyd iteration at the same size.
    The page reports e-means matching 25 Lloyd iterations' test error in about 2 epochs."""
    import exact_lloyd_means_assign_b200 as km
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    Ne, Ke, De, epochs, alpha0 = 1 << 22, 16384, 128, 2, 0.3
    batch = args.emeans_batch
    d = synth.make_workload(4, device=dev, N=Ne, K=Ke)
    X, C0 = d["X"], d["C0"]
    g = torch.Generator(device=dev)
    g.manual_seed(99)
    split_u = torch.rand((epochs, 1, Ke), generator=g, device=dev)
    ws_e = torch.empty(km._load().km_emeans_workspace_size(1, Ke, De, km._dt(X.dtype), 0, batch),
                       dtype=torch.uint8, device=dev)
    ws_f = km.workspace(km.KM_OP_FIT, 1, Ne, Ke, De, X.dtype, dev)
    C = C0.clone()

    def em():
        C.copy_(C0)
        km.km_emeans_fit(X, C, batch, epochs, alpha0, split_u=split_u, ws=ws_e, stream=stream)

    def lloyd():
        C.copy_(C0)
        km.km_fit(X, C, 1, ws=ws_f, stream=stream)

    for _ in range(args.warmup):
        em()
        lloyd()
    with ClockSampler(0) as clk:
        em_ms = _timed(em, args.steps, stream)
        ll_ms = _timed(lloyd, args.steps, stream)
    peak_tf, _, peak_kind = _peaks()
    flop_epoch = 2.0 * Ne * Ke * De
    print(json.dumps({
        "metric": "e-means 2-epoch fit time (vs one Lloyd iteration at the same size)",
        "value": em_ms / 1e3, "unit": "s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": em_ms, "higher_is_better": False, "scaling": "none", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "config": {"workload": "emeans_large_k: B=1 N=2^22 K=16384 d=128 fp16 (8192-comp GMM)",
                   "batch": batch, "epochs": epochs, "alpha0": alpha0, "splitting": True},
        "emeans_ms_per_epoch": em_ms / epochs, "lloyd_ms_per_iteration": ll_ms,
        "lloyd_25_iterations_s": 25 * ll_ms / 1e3,
        "roofline": {"bound": "tensor", "achieved": flop_epoch * epochs / (em_ms * 1e-3) / 1e12,
                     "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": flop_epoch * epochs / (em_ms * 1e-3) / 1e12 / peak_tf,
                     "note": "assignment contraction of every point once per epoch over the whole run",
                     "peak_source": f"{peak_kind} bf16 dense"},
        "clocks": clk.summary(), "device_error": km.km_device_error()}), flush=True)


def run_codebook1d(args):
    """Per-row 1-D codebooks on the weighted-rows workload (4096 rows x 4096 fp16 values):
    k-means++ seeding (K = 16), and encoding every value to its uint8 index against a fitted
    K = 16 codebook. Encoding is bound by HBM: 2 bytes read + 1 byte written per value."""
    import exact_lloyd_means_assign_b200 as km
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    d = synth.make_workload(2, device=dev, K=16)
    X, w = d["X"], d["w"]
    Bc, Nc = X.shape[0], X.shape[1]
    Kc = 16
    C = km.km_init_grid1d(X, Kc)
    km.km_fit(X, C, 30, w=w)
    codes = torch.empty((Bc, Nc), dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    u = torch.rand((Bc, Kc), generator=g, device=dev)

    def enc():
        km.km_encode1d(X, C, codes=codes, stream=stream)

    def pp():
        km.km_init_kmeanspp1d(X, Kc, u, w=w, stream=stream)

    for _ in range(args.warmup):
        enc()
        pp()
    # one encode is shorter than the host-side cost of a call, so the timed unit is a CUDA graph
    # of 20 encode launches (the kernels run back to back, as in a pipeline)
    reps = 20
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            km.km_encode1d(X, C, codes=codes)
    graph.replay()
    steps = _steps_for(graph.replay, args.steps, stream)
    with ClockSampler(0) as clk:
        enc_ms = _timed(graph.replay, steps, stream) / reps
        pp_ms = _timed(pp, max(3, args.steps), stream)
    _, peak_bw, peak_kind = _peaks()
    nbytes = Bc * Nc * (X.element_size() + 1) + Bc * Kc * 4
    print(json.dumps({
        "metric": "1-D codebook encode GB/s (uint8 indices, K=16)", "value": nbytes / enc_ms / 1e6,
        "unit": "GB/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": enc_ms,
        "higher_is_better": True, "scaling": "none", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": "rows_weighted_1d: 4096 rows x 4096 fp16, K=16 fitted codebooks",
                   "l2": "inputs (50 MB) below L2 size; steady-state repeated encode"},
        "values_per_s": Bc * Nc / (enc_ms * 1e-3), "launches_per_graph": reps,
        "kmeanspp_ms": pp_ms,
        "roofline": {"bound": "hbm", "achieved": nbytes / enc_ms / 1e6, "peak": peak_bw, "unit": "GB/s",
                     "frac": nbytes / enc_ms / 1e6 / peak_bw, "algorithmic_bytes": nbytes,
                     "peak_source": peak_kind},
        "clocks": clk.summary(), "device_error": km.km_device_error()}), flush=True)


OOC_WORKLOADS = {
    # name: (synth workload, K override, points per batch element per chunk)
    "batched_assign_bound": (3, None, 16384),
    "single_N33M_K16384": (5, 16384, 1 << 21),
}


def run_out_of_core(args):
    """Out-of-core Lloyd (km_fit_stream): X stays in pinned host memory and every iteration
    streams it through two device chunk buffers. The bound is the host-to-device copy, so the
    roofline line compares the streamed bytes per second with a plain pinned copy of the same
    tensor timed in the same process."""
    import exact_lloyd_means_assign_b200 as km
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    idx, k_over, chunk = OOC_WORKLOADS[args.out_of_core]
    d = synth.make_workload(idx, device=dev, K=k_over)
    Xh = d["X"].cpu().pin_memory()
    C0 = d["C0"]
    del d
    torch.cuda.empty_cache()
    Bo, No, Do = Xh.shape
    Ko = C0.shape[1]
    nbytes = Xh.numel() * Xh.element_size()
    ws = torch.empty(km._load().km_stream_workspace_size(Bo, Ko, Do, km._dt(Xh.dtype), 0, min(chunk, No)),
                     dtype=torch.uint8, device=dev)
    C = C0.clone()
    km.km_fit_stream(Xh, C, args.warmup, chunk, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record()
        km.km_fit_stream(Xh, C, args.steps, chunk, ws=ws)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    buf = torch.empty(Xh.shape, dtype=Xh.dtype, device=dev)
    buf.copy_(Xh, non_blocking=True)
    copy_gbs = 0.0
    for _ in range(3):   # the best of three plain copies: host-side bandwidth varies run to run
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        buf.copy_(Xh, non_blocking=True)
        c1.record()
        torch.cuda.synchronize()
        copy_gbs = max(copy_gbs, nbytes / c0.elapsed_time(c1) / 1e6)
    achieved = nbytes / ms / 1e6
    print(json.dumps({
        "metric": "out-of-core Lloyd iter/s (points in pinned host memory)", "value": 1e3 / ms,
        "unit": "iter/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "none", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": args.out_of_core, "B": Bo, "N": No, "K": Ko, "d": Do,
                   "chunk_points_per_batch": chunk, "x_host_bytes": nbytes},
        "roofline": {"bound": "h2d", "achieved": achieved, "peak": copy_gbs, "unit": "GB/s",
                     "frac": achieved / copy_gbs,
                     "peak_source": "pinned host-to-device copy of X timed in this run"},
        "clocks": clk.summary()}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--out-of-core", choices=sorted(OOC_WORKLOADS), default=None,
                    help="time the streamed fit (points in host memory) instead of the step")
    ap.add_argument("--emeans-batch", type=int, default=4 * 74 * 256,
                    help="mini-batch size of the e-means workload")
    ap.add_argument("--workload", default=None,
                    choices=["tiny_exact", "rows_weighted_1d", "large_k_assign", "contention_update",
                             "emeans", "codebook1d"],
                    help="time one of the other synthetic workloads instead of the headline one")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.out_of_core:
        run_out_of_core(args)
    elif args.workload == "emeans":
        run_emeans(args)
    elif args.workload == "codebook1d":
        run_codebook1d(args)
    elif args.workload:
        run_workload(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
