"""Benchmark: one exact Lloyd iteration (assignment + sort-inverse update) per step.

Workload (the one the headline metric is quoted on): B=32 independent problems, N=65536 points
each, d=128, K=1024 centroids, fp16 points, fp32 centroids; 1024-component Gaussian mixture per
batch (means N(0,1)^128, sigma=0.3), init = K seeded-random points. Inputs (X = 537 MB) are
larger than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --out-of-core {batched_assign_bound,single_N33M_K16384} --steps 5
  python bench.py --workload {tiny_exact,rows_weighted_1d,large_k_assign,contention_update,
                              contention_update_zipf,emeans,codebook1d} [--gpus N]

A step on the GPU = km_assign (tensor-core FlashAssign; the labels and the per-cluster counts,
which is all a Lloyd iteration needs: the per-point distance and the inertia are optional
outputs) + km_update_next (scatter with the scan folded in, then the segmented reduce with the
division fused in,
writing the new centroids, their rounding and norms for the next assignment): exactly one
iteration of km_fit's loop without the objective. The assignment with the inertia
requested is timed separately and reported as "assign_with_inertia_ms".

Timing: W untimed warm-up steps, then blocks of exactly K steps, each bracketed by a barrier and
a device synchronisation and timed with CUDA events on the launching stream. The block is
repeated until about half a second has been timed, so that the clock sampler (nvidia-smi, 100 ms
period) sees the timed region; the reported step time is the median block's, max over ranks.

Multi-GPU: ``--gpus N`` starts N ranks itself (torchrun, one process per GPU) unless it already
runs under a launcher. The headline workload is batch-sharded: every rank runs its own B=32
problems (independent, no data-path collective, weak scaling). ``--workload large_k_assign`` /
``contention_update`` with N > 1 split one problem's points over the ranks (one all-reduce of
the per-cluster partial sums per iteration, strong scaling).

``--impl reference`` times the fp64 CPU oracle on this host (whole iterations of the same
workload when they fit the run's time budget, else whole batch elements) and prints the same
JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import socket
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


def update_bytes(Bw, Nw, Dw, esize):
    """Algorithmic bytes of the sort-inverse update: every point's row gathered once, plus the
    assignment read twice (histogram, scatter) and the sorted order written and read once. The
    per-cluster sums and the new centroids (K-sized) are not counted."""
    return Bw * Nw * Dw * esize + 4 * Bw * Nw * 4


UPDATE_BYTES = update_bytes(B, N, D, 2)
LAUNCHES_PER_STEP = 4   # caug, assign_tc (+ counts), scatter_final (+ scan), segreduce_final
MIN_TIMED_S = 0.5


def _peaks():
    """(burst bf16 TFLOP/s, sustained bf16 TFLOP/s, HBM GB/s, source)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        tf = float(j["bf16_tflops"])
        return tf, float(j.get("bf16_tflops_sustained", tf)), float(j["hbm_gbs"]), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def _kernel_source_hash(files=("km_assign_tc.cuh", "km_common.cuh")):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "exact_lloyd_means_assign_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _profile_traffic(name="assign_tc_batched_assign_bound.md", files=("km_assign_tc.cuh", "km_common.cuh")):
    """DRAM bytes per launch from a committed ncu summary, if it matches this source."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    s = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    if not m or not s or s.group(1) != _kernel_source_hash(files):
        return None
    return float(m.group(1))


def lloyd_roofline(flop, update_bytes, ms_per_iter, peak_tf, peak_gbs):
    """Whole-iteration roofline: the time the assignment's contraction takes at the tensor peak
    plus the time the update's algorithmic bytes take at the HBM peak, over the measured time."""
    ideal_ms = flop / (peak_tf * 1e12) * 1e3 + update_bytes / (peak_gbs * 1e9) * 1e3
    return {"ideal_ms": ideal_ms, "measured_ms": ms_per_iter, "frac": ideal_ms / ms_per_iter,
            "definition": "(flop / tensor peak + update bytes / HBM peak) / time per iteration"}


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


# ---------------------------------------------------------------- launcher

def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_command(gpus, argv):
    """The torchrun command that runs this script as ``gpus`` ranks on this node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]


def _init_pg(backend, dev=None):
    import datetime
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=120)}
    if dev is not None:
        kw["device_id"] = dev
    dist.init_process_group(backend, **kw)
    return dist


def run_launcher_selftest(args):
    """Exercise the multi-rank plumbing without a GPU: every rank joins a gloo group, the ranks
    all-reduce one value and take the max of a per-rank time, rank 0 prints one line."""
    ws, rank, _ = _dist()
    pg = _init_pg("gloo") if ws > 1 else None
    v = torch.tensor([float(rank + 1)])
    t = torch.tensor([0.001 * (rank + 1)], dtype=torch.float64)
    if pg:
        pg.all_reduce(v)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        pg.barrier()
    if rank == 0:
        print(json.dumps({"selftest": True, "n_gpus": ws, "sum_ranks": float(v.item()),
                          "max_time": float(t.item())}), flush=True)
    if pg:
        pg.destroy_process_group()


# ---------------------------------------------------------------- timing helpers

def _timed(fn, steps, stream):
    """Mean device ms of fn() over ``steps`` calls (CUDA events on ``stream``)."""
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        fn()
    t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def _steps_for(fn, steps, stream, min_s=MIN_TIMED_S):
    """At least ``steps``, and enough for ``min_s`` seconds so that the clock sampler (100 ms
    period) sees the timed region."""
    t = _timed(fn, 2, stream)
    return max(steps, int(min_s * 1e3 / max(t, 1e-3)) + 1)


def _median(v):
    v = sorted(v)
    n = len(v)
    return v[n // 2] if n % 2 else 0.5 * (v[n // 2 - 1] + v[n // 2])


def timed_blocks(phases, steps, stream, pg=None, min_s=MIN_TIMED_S):
    """Blocks of exactly ``steps`` steps, each step calling the functions in ``phases`` in order
    with a CUDA event between them; each block is bracketed by a barrier (multi-rank) and a
    device synchronisation. Blocks repeat until ``min_s`` seconds have been timed (at least 3).
    Returns (median block ms per step, [median per-phase ms per step], blocks)."""
    nph = len(phases)
    per_block, per_phase = [], [[] for _ in range(nph)]
    need = 3
    t_total = 0.0
    while len(per_block) < need:
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(steps)]
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        for e in ev:
            e[0].record(stream)
            for j, f in enumerate(phases):
                f()
                e[j + 1].record(stream)
        torch.cuda.synchronize()
        blk = ev[0][0].elapsed_time(ev[-1][nph])
        per_block.append(blk / steps)
        for j in range(nph):
            per_phase[j].append(sum(e[j].elapsed_time(e[j + 1]) for e in ev) / steps)
        t_total += blk * 1e-3
        if len(per_block) == 1:
            need = max(3, math.ceil(min_s / max(blk * 1e-3, 1e-6)))
            # every rank must run the same number of blocks (each starts with a barrier)
            need = _agree_max(need, pg)
    return _median(per_block), [_median(p) for p in per_phase], len(per_block)


def _agree_max(n, pg):
    """The largest of the ranks' values of n (n itself with one process)."""
    if not pg:
        return n
    dev = "cpu" if pg.get_backend() == "gloo" else torch.device("cuda", torch.cuda.current_device())
    t = torch.tensor([n], dtype=torch.int64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return int(t.item())


def _max_over_ranks(vals, pg, dev):
    if not pg:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.tolist()


# ---------------------------------------------------------------- CPU oracle baselines

def cpu_baseline(X, C, budget_s=15.0, w=None):
    """The fp64 oracle (assign + update) on a bounded sample of a batched workload, scaled to
    one full iteration of all of X.

    The sample is the first points of batch element 0, then of element 1, ... (each against its
    own centroids) until about ``budget_s`` seconds of CPU work are reached; only points that
    were actually processed are counted.
    """
    import oracle
    Bx, Nx = X.shape[0], X.shape[1]
    Cb = oracle.round_to_dtype(C[0:1].cpu(), X.dtype)
    n_cal = min(Nx, 1024)
    t = time.perf_counter()
    oracle.assign(oracle.as_f64(X[0:1, :n_cal].cpu()), Cb)
    per_pt = (time.perf_counter() - t) / n_cal
    target = int(min(Bx * Nx, max(n_cal, budget_s * 0.9 / max(per_pt, 1e-9))))
    done, measured, nb = 0, 0.0, 0
    for b in range(Bx):
        if done >= target:
            break
        n = int(min(Nx, target - done))
        Xb = oracle.as_f64(X[b:b + 1, :n].cpu())
        wb = None if w is None else oracle.as_f64(w[b:b + 1, :n].cpu())
        Cb = oracle.round_to_dtype(C[b:b + 1].cpu(), X.dtype)
        t = time.perf_counter()
        ids, _, _, _ = oracle.assign(Xb, Cb, wb)
        oracle.update(Xb, ids, Cb, wb)
        measured += time.perf_counter() - t
        done += n
        nb += 1
    full = measured * (Bx * Nx) / done
    return {"value": 1.0 / full, "unit": "iter/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{done} points of {Bx * Nx} (first points of {nb} batch element(s); assign + "
                      f"update, fp64), {measured:.1f} s measured, scaled by {Bx * Nx / done:.2f} to "
                      f"one full iteration",
            "seconds_measured": measured}


def cpu_update_baseline(X, ids, C, budget_s=10.0):
    """The fp64 oracle's update alone (given assignment) on a bounded sample of points, scaled
    to the whole workload. Returns seconds per full update and the sample description."""
    import oracle
    Nx = X.shape[1]
    n = min(Nx, 1 << 16)
    t = time.perf_counter()
    oracle.update(oracle.as_f64(X[0:1, :n].cpu()), ids[0:1, :n].cpu().numpy(), oracle.as_f64(C[0:1].cpu()))
    per_pt = (time.perf_counter() - t) / n
    n = int(min(Nx, max(n, budget_s * 0.9 / max(per_pt, 1e-12))))
    Xs = oracle.as_f64(X[0:1, :n].cpu())
    ids_s = ids[0:1, :n].cpu().numpy()
    C64 = oracle.as_f64(C[0:1].cpu())
    t = time.perf_counter()
    oracle.update(Xs, ids_s, C64)
    measured = time.perf_counter() - t
    return measured * X.shape[0] * Nx / n, {
        "cores": oracle.threads(), "kind": "oracle",
        "sample": f"update of the first {n} of {X.shape[0] * Nx} points (fp64, given labels), "
                  f"{measured:.2f} s measured, scaled by {X.shape[0] * Nx / n:.2f}"}


# ---------------------------------------------------------------- headline workload

def run_gpu(args):
    import exact_lloyd_means_assign_b200 as km
    import synth

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = _init_pg("nccl", dev) if ws > 1 else None
    # each rank owns its own B=32 problems (independent batches)
    d = synth.make_workload(3, device=dev, seed=1234 + 3 + 1000 * rank)
    X, C = d["X"], d["C0"]
    ws_a = km.workspace(km.KM_OP_ASSIGN, B, N, K, D, X.dtype, dev)
    ws_u = km.workspace(km.KM_OP_UPDATE, B, N, K, D, X.dtype, dev)
    ids = torch.empty((B, N), dtype=torch.int32, device=dev)
    counts = torch.empty((B, K), dtype=torch.int32, device=dev)
    inertia = torch.empty((B,), dtype=torch.float64, device=dev)
    Cx, cn = km.km_prep(C, X.dtype)
    stream = torch.cuda.current_stream()

    def assign():
        km.km_assign(X, Cx, cn, ids=ids, counts=counts, ws=ws_a, stream=stream)

    def update():
        km.km_update_next(X, ids, C, Cx, cn, C_new=C, counts=counts, counts_ready=True, ws=ws_u,
                          stream=stream)

    for _ in range(args.warmup):
        assign()
        update()
    torch.cuda.synchronize()
    with ClockSampler(local) as cs:
        ms_step, (assign_ms, update_ms), blocks = timed_blocks([assign, update], args.steps, stream, pg)
    # the assignment with the objective requested (per-batch inertia), outside the timed steps
    n_in = max(3, min(50, args.steps))
    for _ in range(3):
        km.km_assign(X, Cx, cn, ids=ids, inertia=inertia, ws=ws_a, stream=stream)
    assign_inertia_ms = _timed(lambda: km.km_assign(X, Cx, cn, ids=ids, inertia=inertia, ws=ws_a,
                                                    stream=stream), n_in, stream)
    ms_step, assign_ms, update_ms, assign_inertia_ms = _max_over_ranks(
        [ms_step, assign_ms, update_ms, assign_inertia_ms], pg, dev)
    err = km.km_device_error()

    # end to end through the public host-buffer entry point: H2D of X and C, one iteration,
    # D2H of the new centroids and the inertia, synchronised, every step (device-timed on the
    # stream the call enqueues on)
    Xh = X.cpu().pin_memory()
    Ch = d["C0"].cpu().pin_memory()
    inh = torch.empty((1, B), dtype=torch.float64).pin_memory()
    ws_h = km.workspace(km.KM_OP_FIT_HOST, B, N, K, D, X.dtype, dev, False, 1)
    e2e_steps = max(3, min(20, args.steps))
    km.km_fit_host(Xh, Ch, 1, inertia_host=inh, ws=ws_h, device=dev)
    if pg:
        pg.barrier()
    e2e_ms = _timed(lambda: km.km_fit_host(Xh, Ch, 1, inertia_host=inh, ws=ws_h, device=dev,
                                           stream=stream), e2e_steps, stream)
    (e2e_ms,) = _max_over_ranks([e2e_ms], pg, dev)

    clocks = cs.summary()
    if rank == 0:
        peak_tf, peak_tf_sus, peak_bw, peak_kind = _peaks()
        achieved_tf = ASSIGN_FLOP / (assign_ms * 1e-3) / 1e12
        upd_gbs = UPDATE_BYTES / (update_ms * 1e-3) / 1e9
        line = {
            "metric": METRIC,
            "value": ws * 1e3 / ms_step,
            "unit": "iter/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "N": N, "K": K, "d": D, "iterations_per_step": 1,
                       "init": "K seeded-random points per batch", "l2": "inputs larger than L2 (X = 537 MB)",
                       "parallelism": f"batch-sharded x{ws} (independent problems, no collective)",
                       "timing": f"median of {blocks} blocks of {args.steps} steps"},
            "timed_blocks": blocks,
            "assign_pt_k_per_s": ws * B * N * K / (assign_ms * 1e-3),
            "assign_ms": assign_ms,
            "update_ms": update_ms,
            "assign_with_inertia_ms": assign_inertia_ms,
            "roofline": {"bound": "tensor", "kernel": "assign_tc_kernel (+ caug_kernel, the centroid side of the norm step)",
                         "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": achieved_tf / peak_tf, "frac_of_sustained": achieved_tf / peak_tf_sus,
                         "traffic": _profile_traffic(),
                         "peak_source": f"{peak_kind} bf16 dense, burst (fp16 nominal ratio 1.0)"},
            "update_roofline": {"bound": "hbm", "achieved": upd_gbs, "peak": peak_bw, "unit": "GB/s",
                                "frac": upd_gbs / peak_bw, "algorithmic_bytes": UPDATE_BYTES,
                                "peak_source": peak_kind},
            "lloyd_roofline": lloyd_roofline(ASSIGN_FLOP, UPDATE_BYTES, ms_step, peak_tf, peak_bw),
            "e2e": {"value": ws * 1e3 / e2e_ms, "unit": "iter/s",
                    "h2d_bytes_per_step": B * N * D * 2 + B * K * D * 4,
                    "d2h_bytes_per_step": B * K * D * 4 + B * 8},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps * blocks,
            "clocks": clocks,
            "device_error": err,
        }
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(X, d["C0"], budget_s=args.cpu_budget)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, on the headline workload. A timed
    step is one whole Lloyd iteration of all B=32 problems (assign + update) when ``steps`` of
    them fit about 200 s; otherwise the largest number of whole batch elements that does (the
    value is then scaled to a full iteration, and the line says so)."""
    ws, rank, _ = _dist()
    if rank != 0:
        return
    import oracle
    import synth
    d = synth.make_workload(3, device="cpu")
    X, C = d["X"], d["C0"]
    Bx = X.shape[0]

    def batch_step(b):
        Xb = oracle.as_f64(X[b:b + 1])
        Cb = oracle.round_to_dtype(C[b:b + 1], X.dtype)
        ids, _, _, _ = oracle.assign(Xb, Cb)
        oracle.update(Xb, ids, Cb)

    t = time.perf_counter()
    batch_step(0)                      # calibration (and page-in), not timed
    t_batch = time.perf_counter() - t
    budget = 200.0
    per_step = max(1, min(Bx, int(budget / max(1, args.steps) / max(t_batch, 1e-6))))
    for w_ in range(args.warmup):      # warm-up: one batch element each
        batch_step((w_ + 1) % Bx)
    secs = []
    nxt = 0
    for _ in range(args.steps):
        t = time.perf_counter()
        for _j in range(per_step):
            batch_step(nxt % Bx)
            nxt += 1
        secs.append(time.perf_counter() - t)
    s_step = sum(secs) / len(secs)
    s_iter = s_step * Bx / per_step
    sample = (f"each step = {per_step} whole batch element(s) of {Bx} (N={N}, assign + update, fp64)"
              + ("" if per_step == Bx else f", scaled by {Bx / per_step:.2f} to a full iteration"))
    line = {
        "metric": METRIC, "impl": "reference", "value": 1.0 / s_iter, "unit": "iter/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "N": N, "K": K, "d": D, "iterations_per_step": per_step / Bx},
        "cpu_baseline": {"value": 1.0 / s_iter, "unit": "iter/s", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": 1.0 / s_iter, "unit": "iter/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- other workloads

def _cpu_fit_baseline_rows(X, w, K, iters, budget_s=10.0):
    """The oracle's weighted 1-D fit (grid init, ``iters`` iterations) on whole rows until about
    ``budget_s`` seconds, scaled to all rows. Returns (fits per second of all rows, sample)."""
    import oracle
    rows = 0
    t0 = time.perf_counter()
    Bx = X.shape[0]
    while rows < Bx and time.perf_counter() - t0 < budget_s:
        n = min(Bx - rows, 16)
        Xr = oracle.as_f64(X[rows:rows + n].cpu())
        wr = oracle.as_f64(w[rows:rows + n].cpu())
        oracle.fit(Xr, oracle.grid_init(Xr, K), iters, w=wr, assign_dtype=X.dtype)
        rows += n
    s = time.perf_counter() - t0
    full = s * Bx / rows
    return full, {"cores": oracle.threads(), "kind": "oracle",
                  "sample": f"{rows} of {Bx} rows (grid init + {iters} iterations, fp64), "
                            f"{s:.1f} s measured, scaled by {Bx / rows:.1f}"}


def run_workload(args):
    """The other synthetic workloads of the measurement table, one JSON line each, 1 GPU (or
    point-sharded over N GPUs for the two B=1 ones): tiny_exact (latency, fp32 exact path,
    eager and CUDA-graph replay of a 20-iteration fit), rows_weighted_1d (the fused per-row 1-D
    fit, K=16 and K=8), large_k_assign and contention_update (one Lloyd iteration per step:
    tensor-core roofline for the assignment, HBM roofline for the sort-inverse update), and
    contention_update_zipf (the update alone, fed the mixture's own Zipf component labels so the
    largest segment holds about 16 % of the points). Every line carries the oracle timed on the
    host cores beside it."""
    import exact_lloyd_means_assign_b200 as km
    import synth

    ws_, rank, local = _dist()
    if ws_ > 1:
        if args.workload in ("large_k_assign", "contention_update"):
            return run_point_sharded(args)
        raise SystemExit(f"--workload {args.workload} runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    name = "contention_update" if args.workload == "contention_update_zipf" else args.workload
    wl = synth.WORKLOADS[{w.name: i for i, w in synth.WORKLOADS.items()}[name]]
    peak_tf, peak_tf_sus, peak_bw, peak_kind = _peaks()
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
        for _ in range(args.warmup):
            g.replay()
        with ClockSampler(0) as clk:
            graph, _, blocks = timed_blocks([g.replay], args.steps, stream)
            eager, _, _ = timed_blocks([fit], args.steps, stream)
        import oracle
        t = time.perf_counter()
        oracle.fit(oracle.as_f64(X.cpu()), oracle.as_f64(C0.cpu()), iters, assign_dtype=X.dtype)
        cpu_s = time.perf_counter() - t
        lines.append(dict(base, metric="exact fp32 Lloyd us/iteration (CUDA-core path)",
                          value=graph * 1e3 / iters, unit="us/iter", higher_is_better=False,
                          ms_per_step=graph, timed_blocks=blocks,
                          eager_us_per_iter=eager * 1e3 / iters,
                          config={"workload": wl.name, "B": Bw, "N": Nw, "K": Kw, "d": Dw,
                                  "iterations_per_step": iters, "launch": "CUDA graph of one km_fit call"},
                          roofline={"bound": "latency",
                                    "note": "4.2 MFLOP per iteration; the whole fit is one cooperative "
                                            "launch (fit_small_kernel) with one grid barrier per iteration"},
                          gpu_launches=args.steps * blocks,
                          cpu_baseline={"value": cpu_s * 1e6 / iters, "unit": "us/iter",
                                        "cores": oracle.threads(), "kind": "oracle",
                                        "sample": f"the whole fit ({iters} iterations, fp64), {cpu_s:.2f} s"},
                          clocks=clk.summary()))
    elif wl.name == "rows_weighted_1d":
        for Kw in wl.K:
            d = synth.make_workload(wl.idx, device=dev, K=Kw)
            X, w = d["X"], d["w"]
            Bw, Nw = X.shape[0], X.shape[1]
            iters = d["iters"]
            C = torch.empty((Bw, Kw, 1), dtype=torch.float32, device=dev)

            def fit(it):
                km.km_init_grid1d(X, Kw, C=C, stream=stream)
                km.km_fit(X, C, it, w=w, stream=stream)

            for _ in range(args.warmup):
                fit(iters)
            with ClockSampler(0) as clk:
                ms, _, blocks = timed_blocks([lambda: fit(iters)], args.steps, stream)
                ms0, _, _ = timed_blocks([lambda: fit(0)], args.steps, stream)
            clocks = clk.summary()
            # the once-per-fit sort prologue against HBM: reads the row and its weights
            # (2 + 4 B), writes the sorted values, their indices and two fp64 prefix sums (24 B)
            pro_bytes = Bw * Nw * (X.element_size() + 4 + 24)
            cpu_s, cpu_desc = _cpu_fit_baseline_rows(X, w, Kw, iters)
            lines.append(dict(base, metric="weighted 1-D per-row fit iter/s (all rows)",
                              value=iters * 1e3 / ms, unit="iter/s", ms_per_step=ms, timed_blocks=blocks,
                              config={"workload": wl.name, "B": Bw, "N": Nw, "K": Kw, "d": 1,
                                      "iterations_per_step": iters, "weighted": True, "init": "grid"},
                              prologue_ms=ms0, us_per_iteration=(ms - ms0) * 1e3 / iters,
                              roofline={"bound": "hbm", "kernel": "fit1d_sort_kernel (the prologue)",
                                        "achieved": pro_bytes / (ms0 * 1e-3) / 1e9, "peak": peak_bw,
                                        "unit": "GB/s", "frac": pro_bytes / (ms0 * 1e-3) / 1e9 / peak_bw,
                                        "algorithmic_bytes": pro_bytes, "peak_source": peak_kind,
                                        "note": "the prologue and the iterations (O(K log N) per row, "
                                                "see us_per_iteration) are both issue-bound, at 70-74 % "
                                                "of the instruction issue peak under ncu; the HBM "
                                                "fraction is that of the prologue's bytes"},
                              cpu_baseline=dict(cpu_desc, value=iters / cpu_s, unit="iter/s"),
                              clocks=clocks))
    elif args.workload == "contention_update_zipf":
        d = synth.make_workload(wl.idx, device=dev, labels=True)
        X, C, ids = d["X"], d["C0"], d["labels"]
        Bw, Nw, Dw = X.shape
        Kw = C.shape[1]
        ws_u = km.workspace(km.KM_OP_UPDATE, Bw, Nw, Kw, Dw, X.dtype, dev)
        counts = torch.empty((Bw, Kw), dtype=torch.int32, device=dev)
        C_new = torch.empty_like(C)
        Cx, cn = km.km_prep(C, X.dtype)

        def update():   # the histogram of the labels is part of this update
            km.km_update_next(X, ids, C, Cx, cn, C_new=C_new, counts=counts, ws=ws_u, stream=stream)

        for _ in range(args.warmup):
            update()
        with ClockSampler(0) as clk:
            u_ms, _, blocks = timed_blocks([update], args.steps, stream)
        largest = float(torch.bincount(ids[0].long(), minlength=Kw).max()) / Nw
        ubytes = update_bytes(Bw, Nw, Dw, X.element_size())
        cpu_s, cpu_desc = cpu_update_baseline(X, ids, C)
        lines.append(dict(base, metric="sort-inverse update GB/s (hot-cluster labels)",
                          value=ubytes / (u_ms * 1e-3) / 1e9, unit="GB/s", ms_per_step=u_ms,
                          timed_blocks=blocks,
                          config={"workload": "contention_update_zipf: X of contention_update, ids = the "
                                              "mixture's Zipf(1.1) component labels",
                                  "B": Bw, "N": Nw, "K": Kw, "d": Dw, "largest_segment_frac": largest,
                                  "l2": "inputs larger than L2"},
                          roofline={"bound": "hbm", "kernel": "hist+scatter_final+segreduce_final",
                                    "achieved": ubytes / (u_ms * 1e-3) / 1e9, "peak": peak_bw, "unit": "GB/s",
                                    "frac": ubytes / (u_ms * 1e-3) / 1e9 / peak_bw,
                                    "algorithmic_bytes": ubytes, "peak_source": peak_kind},
                          gpu_launches=3 * args.steps * blocks,
                          cpu_baseline=dict(cpu_desc, value=ubytes / cpu_s / 1e9, unit="GB/s"),
                          clocks=clk.summary(), device_error=km.km_device_error()))
    else:
        d = synth.make_workload(wl.idx, device=dev)
        X, C = d["X"], d["C0"]
        Bw, Nw, Dw = X.shape
        Kw = C.shape[1]
        ws_a = km.workspace(km.KM_OP_ASSIGN, Bw, Nw, Kw, Dw, X.dtype, dev)
        ws_u = km.workspace(km.KM_OP_UPDATE, Bw, Nw, Kw, Dw, X.dtype, dev)
        ids = torch.empty((Bw, Nw), dtype=torch.int32, device=dev)
        counts = torch.empty((Bw, Kw), dtype=torch.int32, device=dev)
        Cx, cn = km.km_prep(C, X.dtype)

        def assign():
            km.km_assign(X, Cx, cn, ids=ids, counts=counts, ws=ws_a, stream=stream)

        def update():
            km.km_update_next(X, ids, C, Cx, cn, C_new=C, counts=counts, counts_ready=True, ws=ws_u,
                              stream=stream)

        for _ in range(args.warmup):
            assign()
            update()
        torch.cuda.synchronize()
        with ClockSampler(0) as clk:
            ms, (a_ms, u_ms), blocks = timed_blocks([assign, update], args.steps, stream)
        flop = 2.0 * Bw * Nw * Kw * Dw
        ubytes = update_bytes(Bw, Nw, Dw, X.element_size())
        cpu = cpu_baseline(X, d["C0"], budget_s=args.cpu_budget) if not args.no_cpu_baseline else None
        line = dict(base, metric="Lloyd iter/s & assign pt·K/s; % roofline", value=1e3 / ms,
                    unit="iter/s", ms_per_step=ms, assign_ms=a_ms, update_ms=u_ms, timed_blocks=blocks,
                    assign_pt_k_per_s=Bw * Nw * Kw / (a_ms * 1e-3),
                    config={"workload": wl.name, "B": Bw, "N": Nw, "K": Kw, "d": Dw,
                            "iterations_per_step": 1, "l2": "inputs larger than L2"},
                    roofline={"bound": "tensor", "kernel": "assign_tc_kernel",
                              "achieved": flop / (a_ms * 1e-3) / 1e12, "peak": peak_tf,
                              "unit": "TFLOP/s", "frac": flop / (a_ms * 1e-3) / 1e12 / peak_tf,
                              "frac_of_sustained": flop / (a_ms * 1e-3) / 1e12 / peak_tf_sus,
                              "traffic": None, "peak_source": f"{peak_kind} bf16 dense, burst"},
                    update_roofline={"bound": "hbm", "achieved": ubytes / (u_ms * 1e-3) / 1e9,
                                     "peak": peak_bw, "unit": "GB/s",
                                     "frac": ubytes / (u_ms * 1e-3) / 1e9 / peak_bw,
                                     "algorithmic_bytes": ubytes, "peak_source": peak_kind},
                    lloyd_roofline=lloyd_roofline(flop, ubytes, ms, peak_tf, peak_bw),
                    gpu_launches=LAUNCHES_PER_STEP * args.steps * blocks, clocks=clk.summary(),
                    device_error=km.km_device_error())
        if cpu:
            line["cpu_baseline"] = cpu
        lines.append(line)
    for l in lines:
        print(json.dumps(l), flush=True)


def run_point_sharded(args):
    """One B=1 workload split over the ranks by points (strong scaling): per step every rank
    assigns its slice and forms partial per-cluster sums, one all-reduce of the partials over
    NCCL, and an identical divide on every rank (``dist.lloyd_step_point_sharded``)."""
    import exact_lloyd_means_assign_b200 as km
    from exact_lloyd_means_assign_b200 import dist as kdist
    import synth

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = _init_pg("nccl", dev)
    wl = synth.WORKLOADS[{w.name: i for i, w in synth.WORKLOADS.items()}[args.workload]]
    d = synth.make_workload(wl.idx, device=dev)           # same seed, same bits on every rank
    X, C0 = d["X"], d["C0"]
    Bw, Nw, Dw = X.shape
    Kw = C0.shape[1]
    s, e = kdist.point_shard(Nw, rank, ws)
    X_local = X[:, s:e].contiguous()
    del X, d
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()
    ops = kdist.LibraryOps(stream)
    C = C0.clone()

    def step():
        nonlocal C
        C, _, _ = kdist.lloyd_step_point_sharded(X_local, C, group=None, ops=ops)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms, _, blocks = timed_blocks([step], args.steps, stream, pg)
    (ms,) = _max_over_ranks([ms], pg, dev)
    clocks = clk.summary()
    if rank == 0:
        peak_tf, peak_tf_sus, _, peak_kind = _peaks()
        flop = 2.0 * Bw * Nw * Kw * Dw
        print(json.dumps({
            "metric": "Lloyd iter/s & assign pt·K/s; % roofline", "value": 1e3 / ms, "unit": "iter/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic", "timed_blocks": blocks,
            "config": {"workload": wl.name, "B": Bw, "N": Nw, "K": Kw, "d": Dw, "iterations_per_step": 1,
                       "parallelism": f"point-sharded x{ws}: one all-reduce of per-cluster partial sums "
                                      f"per iteration (NCCL)"},
            "roofline": {"bound": "tensor", "achieved": flop / (ms * 1e-3) / 1e12 / ws,
                         "peak": peak_tf, "unit": "TFLOP/s per GPU",
                         "frac": flop / (ms * 1e-3) / 1e12 / ws / peak_tf,
                         "note": "whole step (assign, update, exchange) against the contraction",
                         "peak_source": f"{peak_kind} bf16 dense, burst"},
            "clocks": clocks, "device_error": km.km_device_error()}), flush=True)
    pg.barrier()
    pg.destroy_process_group()


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

    def em(st=stream):
        C.copy_(C0)
        km.km_emeans_fit(X, C, batch, epochs, alpha0, split_u=split_u, ws=ws_e, stream=st)

    def lloyd():
        C.copy_(C0)
        km.km_fit(X, C, 1, ws=ws_f, stream=stream)

    for _ in range(args.warmup):
        em()
        lloyd()
    # the whole fit is stream-ordered, so it is captured once and replayed (no launch gaps
    # between the mini-batches' kernels)
    g_em = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_em):
        em(None)        # the current stream is the capture stream here
    g_em.replay()
    with ClockSampler(0) as clk:
        em_ms, _, blocks = timed_blocks([g_em.replay], args.steps, stream)
        em_eager_ms, _, _ = timed_blocks([em], args.steps, stream)
        ll_ms, _, _ = timed_blocks([lloyd], args.steps, stream)
    peak_tf, _, _, peak_kind = _peaks()
    flop_epoch = 2.0 * Ne * Ke * De
    print(json.dumps({
        "metric": "e-means 2-epoch fit time (vs one Lloyd iteration at the same size)",
        "value": em_ms / 1e3, "unit": "s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": em_ms, "higher_is_better": False, "scaling": "none", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic", "timed_blocks": blocks,
        "config": {"workload": "emeans_large_k: B=1 N=2^22 K=16384 d=128 fp16 (8192-comp GMM)",
                   "batch": batch, "epochs": epochs, "alpha0": alpha0, "splitting": True},
        "emeans_ms_per_epoch": em_ms / epochs, "emeans_eager_ms": em_eager_ms,
        "launch": "CUDA graph of one km_emeans_fit call", "lloyd_ms_per_iteration": ll_ms,
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

    def pp():
        km.km_init_kmeanspp1d(X, Kc, u, w=w, stream=stream)

    for _ in range(args.warmup):
        km.km_encode1d(X, C, codes=codes, stream=stream)
        pp()
    # one encode is shorter than the host-side cost of a call, so the timed unit is a CUDA graph
    # of 20 encode launches (the kernels run back to back, as in a pipeline)
    reps = 20
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            km.km_encode1d(X, C, codes=codes)
    graph.replay()
    with ClockSampler(0) as clk:
        enc_ms, _, blocks = timed_blocks([graph.replay], args.steps, stream)
        pp_ms, _, _ = timed_blocks([pp], args.steps, stream, min_s=0.2)
    enc_ms /= reps
    _, _, peak_bw, peak_kind = _peaks()
    nbytes = Bc * Nc * (X.element_size() + 1) + Bc * Kc * 4
    print(json.dumps({
        "metric": "1-D codebook encode GB/s (uint8 indices, K=16)", "value": nbytes / enc_ms / 1e6,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": enc_ms,
        "higher_is_better": True, "scaling": "none", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic", "timed_blocks": blocks,
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


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
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
                             "contention_update_zipf", "emeans", "codebook1d"],
                    help="time one of the other synthetic workloads instead of the headline one")
    ap.add_argument("--launcher-selftest", action="store_true",
                    help="run only the multi-rank plumbing (gloo, no GPU) and print one line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks ourselves
        return subprocess.call(relaunch_command(args.gpus, argv))
    if args.launcher_selftest:
        run_launcher_selftest(args)
    elif args.out_of_core:
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
    return 0


if __name__ == "__main__":
    sys.exit(main())
