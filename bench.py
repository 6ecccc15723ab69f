"""Benchmark: exact Lloyd K-Means iterations per second on B200.

One step = one Lloyd iteration (FlashAssign + Sort-Inverse Update) over the
whole point set of the workload (default: N=1,048,576 points, D=128, K=1024,
bf16, a 1024-component Gaussian mixture).  Inputs are resident in device
memory before the timed region; X (256 MiB) is larger than the 126 MB L2, so
no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line (rank 0).  With torchrun (N > 1) every rank runs an
independent replica problem (own seed) and the line reports the whole-job
rate: iterations of all ranks / max-over-ranks device time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, init_rows, make_points, make_problem  # noqa: E402

METRIC = "Lloyd iters/sec and assign GFLOP/s (% bf16 tensor peak), update GB/s (% HBM)"
UNIT = "iters/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Sources each timed kernel is built from: a recorded ncu traffic figure is
# used only while these files are unchanged.
KERNEL_SOURCES = {
    "k_assign": ("k_assign.cu", "km_ptx.cuh", "km_internal.h"),
    "update": ("k_update.cu", "k_sort.cu", "km_rows.cuh", "km_ptx.cuh", "km_internal.h"),
}


def kernel_source_sha(kernel: str = "k_assign") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "means_clustering_flashassign_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha(kernel)
    for line in open(path):
        m = re.match(r"\|\s*(\S+)\s*\|\s*(\S+)\s*\|\s*([0-9.eE+]+)\s*\|\s*([0-9a-f]+)\s*\|", line)
        if m and m.group(1) == kernel and m.group(2) == workload and m.group(4) == sha:
            return float(m.group(3))
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(world, v: float, device="cuda") -> float:
    """The slowest rank's time: every rank contributes, every rank gets it."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(steps: int, world: int, ms_max: float) -> float:
    """Whole-job iterations per second: every rank runs `steps` iterations of
    its own replica problem; the job takes as long as the slowest rank."""
    return steps * world / (ms_max * 1e-3)


def update_bytes(wl) -> float:
    """Algorithmic bytes of one update: read X once, the assignment vector, the
    permutation written and read once, the centroids and counts written."""
    es = 2 if wl.dtype == "bf16" else 4
    N, D, K = wl.N * wl.B, wl.D, wl.K * wl.B
    return N * D * es + 4 * N + 8 * N + 4 * K * D + 4 * K


def assign_flops(wl) -> float:
    return 2.0 * wl.B * wl.N * wl.K * wl.D


def cpu_baseline(wl, X, C0, sample: int, iters: int):
    """The oracle as it stands, on host cores, over a seeded row sample."""
    import oracle
    n = min(sample, wl.N)
    g = torch.Generator().manual_seed(1234)
    rows = torch.randperm(wl.N, generator=g)[:n]
    Xs = X.reshape(-1, wl.D)[rows.to(X.device)].cpu() if wl.B == 1 else X[0].cpu()
    Cs = (C0 if wl.B == 1 else C0[0]).cpu()
    t0 = time.perf_counter()
    oracle.fit(Xs, Cs, iters, mirror=wl.dtype)
    dt = time.perf_counter() - t0
    per_iter_full = dt / iters * (wl.N * wl.B / Xs.shape[0])
    return {"value": 1.0 / per_iter_full, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{Xs.shape[0]} of {wl.N * wl.B} points x {iters} iterations, all K={wl.K} centroids, "
                      f"{dt:.1f} s; rate scaled linearly to the full point count"}


def run_ours(args, world, rank, local):
    import means_clustering_flashassign_b200 as km
    wl = WORKLOADS[args.workload]
    if wl.host_resident:
        if world > 1:
            raise SystemExit("the host-resident workload runs on one GPU")
        return run_host_resident(args, wl, km)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    X, C0, _ = make_problem(wl, seed=args.seed + rank, device=dev)
    X, C0 = X.contiguous(), C0.contiguous()
    torch.cuda.synchronize()
    # warm-up: W iterations through the same entry point
    km.fit_timed(X, C0, args.warmup)
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(world)
        l0 = km.launch_count()
        e0.record(stream)
        r = km.fit_timed(X, C0, args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        launches = km.launch_count() - l0
    barrier(world)
    ms_call = e0.elapsed_time(e1)  # whole call incl. one-time prep and host sync
    ms = r["iters_ms"]             # device time of exactly the timed iterations
    ms_max = max_over_ranks(world, ms)
    # Phase split from a second fit of the same problem, outside the timed
    # region: its events between the assignment and the update stop those two
    # kernels from overlapping their launch, so it is taken apart from `value`.
    phase = km.fit_profile(X, C0, args.steps)["phase_ms"]
    assign_ms = float(phase[:, 0].mean())
    update_ms = float(phase[:, 1].mean())
    pk, pk_kind = peaks()
    af = assign_flops(wl)
    ub = update_bytes(wl)
    a_tf = af / (assign_ms * 1e-3) / 1e12
    u_gbs = ub / (update_ms * 1e-3) / 1e9
    res = None
    if rank == 0:
        value = job_rate(args.steps, world, ms_max)
        dominant_assign = assign_ms >= update_ms
        roof = ({"bound": "tensor", "kernel": "k_assign", "achieved": round(a_tf, 2), "peak": pk["bf16_tflops"],
                 "unit": "TFLOP/s", "frac": round(a_tf / pk["bf16_tflops"], 4),
                 "peak_kind": f"{pk_kind} bf16 burst",
                 "traffic": recorded_traffic("k_assign", wl.name),
                 "algorithmic_per_launch": af}
                if dominant_assign else
                {"bound": "hbm", "kernel": "update", "achieved": round(u_gbs, 1), "peak": pk["hbm_gbs"],
                 "unit": "GB/s", "frac": round(u_gbs / pk["hbm_gbs"], 4), "peak_kind": f"{pk_kind} copy",
                 "traffic": recorded_traffic("update", wl.name), "algorithmic_per_launch": ub})
        res = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "N": wl.N, "D": wl.D, "K": wl.K, "B": wl.B,
                       "mixture": f"{wl.comps or wl.K} comps, centers {wl.centers}, sigma {wl.sigma}, {wl.weights}",
                       "l2": "inputs larger than L2 (X = %.0f MiB)" % (X.numel() * X.element_size() / 2**20),
                       "parallelism": "replicas" if world > 1 else "single"},
            "phases": {"assign_ms": round(assign_ms, 4), "assign_tflops": round(a_tf, 2),
                       "assign_frac_of_bf16_peak": round(a_tf / pk["bf16_tflops"], 4),
                       "update_ms": round(update_ms, 4), "update_gbs": round(u_gbs, 1),
                       "update_frac_of_hbm": round(u_gbs / pk["hbm_gbs"], 4),
                       "update_algorithmic_bytes": ub, "assign_algorithmic_flops": af},
            "roofline": roof,
            "gpu_launches": int(launches),
            "ms_call": round(ms_call, 4),
            "clocks": clk.summary(),
        }
        if world == 1 and args.tile_sweep:
            res["tile_sweep"] = tile_sweep(wl, X, C0, km)
        if world == 1 and args.ablation and wl.B == 1:
            res["ablation"] = ablation(wl, X, C0, km, assign_ms, update_ms)
        if world == 1 and not args.no_e2e:
            res["e2e"] = e2e(args, wl, X, C0, km)
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl, X, C0, args.cpu_sample, 2)
    return res


def _event_ms(fn, reps=3):
    """Median CUDA-event time of fn() on the current stream."""
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return sorted(ts)[len(ts) // 2]


def ablation(wl, X, C0, km, assign_ms, update_ms):
    """The method against the two strategies it replaces, on the same device
    and inputs: materialised distances (library GEMM writes the N x K scores,
    an argmin kernel reads them back; rows chunked so the scores take at most
    8 GiB) and the atomic-scatter update.  Baseline times are CUDA-event
    medians of 3 calls after one warm-up; the method's are the bench's phase
    times (kernel only, norms precomputed once per fit)."""
    chunk = int(max(1, min(wl.N, (8 << 30) // (4 * wl.K), ((1 << 31) - 1) // wl.K)))
    km.ablation_assign_materialized(X, C0, chunk_rows=chunk)  # warm-up (loads cuBLAS)
    torch.cuda.synchronize()
    mat_ms = _event_ms(lambda: km.ablation_assign_materialized(X, C0, chunk_rows=chunk))
    idx, _, _ = km.assign(X, C0)
    C = C0.float().clone()
    km.ablation_update_atomic(X, idx, C)
    torch.cuda.synchronize()
    atom_ms = _event_ms(lambda: km.ablation_update_atomic(X, idx, C))
    return {"assign_flash_ms": round(assign_ms, 4), "assign_materialized_ms": round(mat_ms, 4),
            "assign_speedup": round(mat_ms / assign_ms, 2), "materialized_chunk_rows": chunk,
            "materialized_scores_bytes": int(wl.N) * wl.K * 4,
            "update_sort_inverse_ms": round(update_ms, 4), "update_atomic_ms": round(atom_ms, 4),
            "update_speedup": round(atom_ms / update_ms, 2)}


def tile_sweep(wl, X, C0, km, iters=5):
    """The static shape -> tiling chooser against every tiling that fits
    (forced with KM_ASSIGN_TILE): assignment-kernel time of each (median of
    the per-iteration phase times of one fit), the chooser's loss against the
    fastest, and the time to plan vs the time the sweep took."""
    dt = km.BF16 if wl.dtype == "bf16" else km.F32
    t0 = time.perf_counter()
    chosen = km.plan(km.OP_FIT, wl.B, wl.N, wl.D, wl.K, dt)
    plan_s = time.perf_counter() - t0

    def assign_ms():
        r = km.fit_profile(X, C0, iters)
        # the first objective depends only on X and C0: every tiling must agree
        j0 = r["objective"].reshape(-1, iters)[:, 0].double().sum().item()
        return float(sorted(float(v) for v in r["phase_ms"][:, 0])[iters // 2]), j0

    os.environ.pop("KM_ASSIGN_TILE", None)
    static_ms, j_ref = assign_ms()
    results = []
    t0 = time.perf_counter()
    for pair in (0, 1):
        for bn in (64, 128, 256):
            for xb in range(1, 9):
                for cs in (2, 3, 4):
                    os.environ["KM_ASSIGN_TILE"] = f"{pair},{bn},{xb},{cs}"
                    try:
                        km.workspace_size(km.OP_FIT, wl.B, wl.N, wl.D, wl.K, dt)
                    except km.KMError:
                        continue  # does not fit, or not a tiling for this shape
                    ms, j0 = assign_ms()
                    results.append({"pair": pair, "BN": bn, "XB": xb, "CS": cs, "assign_ms": round(ms, 4),
                                    "objective_ok": abs(j0 - j_ref) <= 1e-6 * abs(j_ref)})
    sweep_s = time.perf_counter() - t0
    os.environ.pop("KM_ASSIGN_TILE", None)
    best = min(results, key=lambda r: r["assign_ms"])
    # the chosen tiling's own entry in the sweep (same conditions as the rest)
    mine = next(r for r in results if all(r[k] == chosen[k] for k in ("pair", "BN", "XB", "CS")))
    return {"chosen": {k: chosen[k] for k in ("pair", "BN", "XB", "CS")}, "chosen_assign_ms": mine["assign_ms"],
            "chosen_unforced_assign_ms": round(static_ms, 4), "best": best,
            "chooser_loss_pct": round(100.0 * (mine["assign_ms"] - best["assign_ms"]) / best["assign_ms"], 2),
            "tilings_tried": len(results), "all_objectives_agree": all(r["objective_ok"] for r in results),
            "plan_seconds": plan_s, "sweep_seconds": round(sweep_s, 2),
            "all": results}


def h2d_link_gbs(src: torch.Tensor, dev) -> float:
    """Pinned host -> device copy bandwidth of this machine (best of 5, CUDA events)."""
    dst = torch.empty(src.shape, dtype=src.dtype, device=dev)
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, src.numel() * src.element_size() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del dst
    return best


def run_host_resident(args, wl, km):
    """The out-of-core workload: X lives in pinned host memory and every
    iteration streams it to the device in chunks (copies overlapped with the
    assignment and update of the previous chunk).  The step is one Lloyd
    iteration over all N points through km_fit_host; the host link, not a
    kernel, bounds it, so the roofline reports host->device bytes against the
    pinned copy bandwidth measured here."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    chunk = 16 << 20
    Xh = torch.empty((wl.N, wl.D), dtype=wl.torch_dtype, pin_memory=True)
    make_points(wl, seed=args.seed, device=dev, out=Xh)
    sel = init_rows(wl, args.seed, dev).cpu()
    C0 = Xh[sel].to(dev).contiguous()
    torch.cuda.synchronize()
    link = h2d_link_gbs(Xh[:chunk], dev)
    km.fit_host(Xh, C0, args.warmup, chunk)
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        l0 = km.launch_count()
        t0 = time.perf_counter()
        r = km.fit_host(Xh, C0, args.steps, chunk)
        Cout = r["C"].cpu()
        dt = time.perf_counter() - t0
        launches = km.launch_count() - l0
    del Cout
    value = args.steps / dt
    xbytes = wl.N * wl.D * Xh.element_size()
    achieved = xbytes * args.steps / dt / 1e9
    h2d = xbytes + C0.numel() * C0.element_size() / args.steps
    d2h = 8 + wl.K * wl.D * 4 / args.steps
    res = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "N": wl.N, "D": wl.D, "K": wl.K, "B": wl.B,
                   "mixture": f"{wl.comps or wl.K} comps, centers {wl.centers}, sigma {wl.sigma}, {wl.weights}",
                   "x": "pinned host memory (%.0f GiB), streamed in %d-row chunks every iteration"
                        % (xbytes / 2**30, chunk),
                   "l2": "inputs larger than L2", "parallelism": "single"},
        "roofline": {"bound": "h2d", "kernel": "km_fit_host stream", "achieved": round(achieved, 1),
                     "peak": round(link, 1), "unit": "GB/s", "frac": round(achieved / link, 4),
                     "peak_kind": "pinned host->device copy measured in this run (best of 5, 16M-row chunk)",
                     "traffic": None, "algorithmic_per_launch": xbytes},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h),
                "how": "the step itself is end to end: X streamed from pinned host memory, centroids read back"},
        "objective": [float(v) for v in r["objective"]],
    }
    if not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, Xh, C0, min(args.cpu_sample, 1 << 18), 1)
    return res


def e2e(args, wl, X, C0, km):
    """Same metric through the public API with host buffers: every iteration
    streams X from pinned host memory (chunks overlapped with compute), and
    the objective history and final centroids are read back to the host."""
    Xh = X.reshape(-1, wl.D).cpu().pin_memory() if wl.B == 1 else None
    if Xh is None:
        return None
    chunk = max(1, wl.N // 4)
    C0d = C0.contiguous()
    km.fit_host(Xh, C0d, 1, chunk)  # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    r = km.fit_host(Xh, C0d, args.steps, chunk)
    Cout = r["C"].cpu()
    dt = time.perf_counter() - t0
    del Cout
    h2d = wl.N * wl.D * X.element_size() + C0.numel() * C0.element_size() / args.steps
    d2h = 8 + wl.K * wl.D * 4 / args.steps
    return {"value": round(args.steps / dt, 3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "chunk_rows": chunk,
            "how": "km_fit_host: X streamed from pinned host memory every iteration, wall clock around the call"}


def run_reference(args, world, rank):
    """The oracle (plain float64 C on the host cores) on a bounded sample."""
    if rank != 0:
        return None
    import oracle
    wl = WORKLOADS[args.workload]
    X, C0, _ = make_problem(wl.with_(N=min(wl.N, args.cpu_sample), K=wl.K) if wl.B == 1 else wl.with_(B=1),
                            seed=args.seed, device="cpu")
    n = X.shape[0] if wl.B == 1 else X.shape[1]
    Xs = X if wl.B == 1 else X[0]
    Cs = C0 if wl.B == 1 else C0[0]
    oracle.fit(Xs, Cs, args.warmup and 1, mirror=wl.dtype)
    t0 = time.perf_counter()
    oracle.fit(Xs, Cs, args.steps, mirror=wl.dtype)
    dt = time.perf_counter() - t0
    per_iter_full = dt / args.steps * (wl.N * wl.B / n)
    value = 1.0 / per_iter_full
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_iter_full * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "N": wl.N, "D": wl.D, "K": wl.K, "B": wl.B},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{n} of {wl.N * wl.B} points, all K={wl.K} centroids, {args.steps} "
                                       f"iterations in {dt:.1f} s; rate scaled linearly to the full point count"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="1m_k1024", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-sample", type=int, default=1 << 20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tile-sweep", action="store_true",
                    help="also time every assignment tiling that fits against the static choice")
    ap.add_argument("--ablation", action="store_true",
                    help="also time the materialised-distance and atomic-scatter baselines")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, world, rank)
    else:
        world, rank, local = dist_setup(args.gpus)
        res = run_ours(args, world, rank, local)
        if world > 1:
            torch.distributed.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
