"""Benchmark: exact Lloyd K-Means iterations per second on B200.

One step = one Lloyd iteration (FlashAssign + Sort-Inverse Update) over the
whole point set of the workload.  The default workload is the largest
device-resident configuration: N=4,194,304 points, D=128, K=16,384, bf16,
a Gaussian mixture with Zipf(1.2) component weights (a few hot clusters).
Inputs are resident in device memory before the timed region; X (1 GiB) is
far larger than the 126 MB L2, so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Timing: W warm-up iterations, then the K-step fit is repeated until the
timed region lasts at least --min-timed-s seconds (1 s by default), so the
clock samples fall under load; each repetition is timed on the device (CUDA
events around its iterations only) and the median repetition gives `value`
and `ms_per_step`.  `value_call` is the same rate over the whole call
(operand preparation, launches and the host synchronisation included).

Prints one JSON line (rank 0).  With torchrun (N > 1) the ranks run one
problem sharded by rows (data-parallel Lloyd: each rank assigns and sums its
own rows, one NCCL all-reduce of float64 sums, counts and objective per
iteration); every rank holds N points (weak scaling), and `value` counts
Lloyd iterations over N points, i.e. steps x ranks / max-over-ranks time.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, init_rows, make_points, make_problem, pool_workload  # noqa: E402

METRIC = "Lloyd iters/sec and assign GFLOP/s (% bf16 tensor peak), update GB/s (% HBM)"
UNIT = "iters/s"
DEFAULT_WORKLOAD = "4m_k16384_zipf"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


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
    """DRAM bytes per launch of `kernel` on `workload` from the record that
    `--record-traffic` wrote from an ncu capture, if that capture was taken on
    the current kernel sources (else None)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f)
    sha = kernel_source_sha(kernel)
    for e in rec.get("entries", []):
        if e["kernel"] == kernel and e["workload"] == workload and e["sources"] == sha:
            return float(e["bytes_per_launch"])
    return None


def record_traffic(csv_path: str, kernel: str, workload: str, scale: float, command: str) -> dict:
    """Read dram__bytes_read.sum + dram__bytes_write.sum of the launches of
    `kernel` from an ncu `--page raw --csv` export, average them per launch,
    multiply by `scale` (full-size units / captured units; 1 for a capture of
    the full workload) and store the figure with the hash of the kernel's
    current sources in profiles/traffic.json."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    head = rows[0]
    ik = head.index("Kernel Name")
    cols = [head.index(m) for m in ("dram__bytes_read.sum", "dram__bytes_write.sum")]
    units = rows[1] if rows[1][cols[0]] in ("byte", "Kbyte", "Mbyte", "Gbyte") else None
    mult = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    vals = []
    for r in rows[1 + (units is not None):]:
        if kernel not in r[ik]:
            continue
        tot = 0.0
        for c in cols:
            tot += float(r[c].replace(",", "")) * (mult[units[c]] if units else 1.0)
        vals.append(tot)
    if not vals:
        raise SystemExit(f"no launch of {kernel} in {csv_path}")
    entry = {"kernel": kernel, "workload": workload, "bytes_per_launch": round(sum(vals) / len(vals) * scale),
             "launches_captured": len(vals), "scale": scale, "sources": kernel_source_sha(kernel),
             "command": command}
    rec = {"entries": []}
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    rec["entries"] = [e for e in rec["entries"] if not (e["kernel"] == kernel and e["workload"] == workload)]
    rec["entries"].append(entry)
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    return entry


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu = gpu_index
        self.period = period_ms
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
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
        sm, pw, mx, reasons = [], [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                pw.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "period_ms": self.period, "power_w_median": statistics.median(pw) if pw else None}


def dist_setup(n_gpus, backend: str = "nccl", same_device: bool = False):
    """One process per GPU (rank r on cuda:LOCAL_RANK) over NCCL.  For a
    single-GPU smoke run of the multi-rank path, `same_device` puts every
    rank on cuda:0 and `backend` "gloo" exchanges through host copies (the
    ranks' kernels never wait on one another)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = 0 if same_device else int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(world, v: float, device="cuda") -> float:
    """The slowest rank's value: every rank contributes, every rank gets it."""
    if world == 1:
        return v
    if torch.distributed.get_backend() == "gloo":
        device = "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(steps: int, world: int, ms_max: float) -> float:
    """Whole-job rate in iterations over one rank's N points per second:
    every rank processes its N points `steps` times (its own replica, or its
    shard of the data-parallel problem); the job takes as long as the slowest
    rank."""
    return steps * world / (ms_max * 1e-3)


def shard_rows(n_per_rank: int, world: int, rank: int) -> slice:
    """Rows of the world * n_per_rank-point problem that rank `rank` holds."""
    return slice(rank * n_per_rank, (rank + 1) * n_per_rank)


def repeats_for(min_timed_s: float, est_ms: float) -> int:
    """Repetitions of the K-step fit that make the timed region last at least
    min_timed_s, given one repetition's estimated milliseconds (from an
    untimed fit that runs before the clock settles under the power cap,
    hence a 15 % margin)."""
    return max(1, int(math.ceil(min_timed_s * 1.15e3 / max(est_ms, 1e-3))))


def update_bytes(wl) -> float:
    """Algorithmic bytes of one update: read X once, the assignment vector, the
    permutation written and read once, the centroids and counts written."""
    es = 2 if wl.dtype == "bf16" else 4
    N, D, K = wl.N * wl.B, wl.D, wl.K * wl.B
    return N * D * es + 4 * N + 8 * N + 4 * K * D + 4 * K


def assign_flops(wl) -> float:
    return 2.0 * wl.B * wl.N * wl.K * wl.D


def workload_config(wl, world: int, parallelism: str) -> dict:
    """The `config` object of the JSON line; the same for both arms."""
    es = 2 if wl.dtype == "bf16" else 4
    xb = wl.B * wl.N * wl.D * es
    cfg = {"workload": wl.name, "N": wl.N, "D": wl.D, "K": wl.K, "B": wl.B, "dtype": wl.dtype,
           "mixture": f"{wl.comps or wl.K} comps, centers {wl.centers}, sigma {wl.sigma}, {wl.weights}",
           "init": "C0 = X rows at the first K entries of a seeded permutation",
           "l2": "inputs larger than L2, no flush (X = %.0f MiB per rank)" % (xb / 2**20) if xb > (126 << 20)
           else "X = %.1f MiB fits in L2: kept resident between steps" % (xb / 2**20),
           "parallelism": parallelism, "ranks": world}
    if wl.host_resident:
        cfg["x"] = "pinned host memory, streamed in 16M-row chunks every iteration"
    if wl.pool_rows:
        cfg["x"] = (f"{wl.N} rows never held whole: streamed in 16M-row chunks from a {wl.pool_rows}-row pinned "
                    f"pool, row i = pool row i mod {wl.pool_rows}")
    return cfg


def make_inputs(wl, seed: int, device):
    """The workload's X and C0 (the same tensors for the same seed and device)."""
    X, C0, _ = make_problem(wl, seed=seed, device=device)
    return X.contiguous(), C0.contiguous()


def make_dp_shard(wl, seed: int, world: int, rank: int, device):
    """This rank's rows of the world * N-point data-parallel problem, and the
    shared C0 (rows of the whole problem at the first K entries of a seeded
    permutation, regenerated chunk by chunk on every rank)."""
    whole = wl.with_(N=wl.N * world)
    rows = shard_rows(wl.N, world, rank)
    X = torch.empty((wl.N, wl.D), dtype=wl.torch_dtype, device=device)
    make_points(whole, seed=seed, device=device, rows=rows, out=X)
    sel = init_rows(whole, seed, device)
    C0 = torch.empty((wl.K, wl.D), dtype=wl.torch_dtype, device=device)
    chunk = 1 << 22
    for c0 in range(0, whole.N, chunk):
        m = (sel >= c0) & (sel < c0 + chunk)
        if not bool(m.any()):
            continue
        part = torch.empty((min(chunk, whole.N - c0), wl.D), dtype=wl.torch_dtype, device=device)
        make_points(whole, seed=seed, device=device, rows=slice(c0, c0 + part.shape[0]), out=part)
        C0[m] = part[sel[m] - c0]
    return X.contiguous(), C0.contiguous()


def oracle_rows(wl, X, C0, target_s: float, iters: int, seed: int = 1234):
    """Seeded uniform row sample of the workload sized so that `iters` oracle
    iterations over it take about target_s seconds of host work (a short probe
    of one iteration on a few rows calibrates the size).  Returns the sample
    rows (CPU) and the centroids (CPU)."""
    import oracle
    Xf = X.reshape(-1, wl.D)
    n_all = Xf.shape[0]
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_all, generator=g)
    Cs = (C0 if C0.dim() == 2 else C0[0]).cpu()
    # probe: double the rows until one iteration takes 0.3 s (or all rows),
    # so thread start-up does not dominate the per-row estimate
    probe = min(n_all, 64)
    while True:
        Xp = Xf[perm[:probe].to(Xf.device)].cpu()
        t0 = time.perf_counter()
        oracle.fit(Xp, Cs, 1, mirror=wl.dtype)
        el = time.perf_counter() - t0
        if el >= 0.3 or probe >= n_all:
            break
        probe = min(n_all, probe * 2)
    per_row = el / probe
    n = int(min(n_all, max(probe, target_s / max(per_row * iters, 1e-12))))
    return Xf[perm[:n].to(Xf.device)].cpu(), Cs


def oracle_sample(wl, X, C0, target_s: float, iters: int):
    """The oracle as it stands on a calibrated sample: returns (seconds per
    iteration scaled to the full point count, sample rows, seconds spent)."""
    import oracle
    Xs, Cs = oracle_rows(wl, X, C0, target_s, iters)
    t0 = time.perf_counter()
    oracle.fit(Xs, Cs, iters, mirror=wl.dtype)
    dt = time.perf_counter() - t0
    return dt / iters * (wl.N * wl.B / Xs.shape[0]), Xs.shape[0], dt


def cpu_baseline(wl, X, C0, target_s: float, iters: int = 1):
    import oracle
    s_per_iter, n, dt = oracle_sample(wl, X, C0, target_s, iters)
    return {"value": 1.0 / s_per_iter, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} of {wl.N * wl.B} points (seeded uniform sample) x {iters} iteration(s), all "
                      f"K={wl.K} centroids, {dt:.1f} s of host work; rate scaled linearly to the full point count"}


def _median(v):
    return statistics.median(v)


def run_ours(args, world, rank, local):
    import means_clustering_flashassign_b200 as km
    wl = WORKLOADS[args.workload]
    if wl.host_resident:
        if world > 1:
            raise SystemExit("the host-resident workload runs on one GPU")
        return run_host_resident(args, wl, km)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dp = world > 1 and args.parallelism == "dp"
    if dp and wl.B != 1:
        raise SystemExit("data-parallel mode shards one problem; use --parallelism replicas for batched workloads")
    parallelism = f"dp{world}" if dp else ("replicas" if world > 1 else "single")
    if dp:
        X, C0 = make_dp_shard(wl, args.seed, world, rank, dev)
    else:
        X, C0 = make_inputs(wl, args.seed + rank, dev)
    torch.cuda.synchronize()

    def one_fit(iters):
        """(device ms of the iterations, device ms of the whole call)."""
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dp:
            c0.record()
            km.fit_data_parallel(X, C0, iters, sync_objective=False)
            c1.record()
            torch.cuda.synchronize()
            ms = c0.elapsed_time(c1)
            return ms, ms
        c0.record()
        r = km.fit_timed(X, C0, iters)
        c1.record()
        torch.cuda.synchronize()
        return r["iters_ms"], c0.elapsed_time(c1)

    one_fit(args.warmup)
    # Untimed K-step fits size the repeats: the warm-up call also
    # carries the first call's module loading and workspace set-up, which
    # would inflate the estimate and shorten the timed region.  A repeat
    # costs the larger of its device time and its wall time (short fits are
    # bound by the host's launch and synchronisation cost).
    # The smaller of two such fits: the first can still carry allocator
    # growth for the call's outputs.
    ests = []
    for _ in range(2):
        t_cal = time.perf_counter()
        _, e = one_fit(args.steps)
        ests.append(max(e, (time.perf_counter() - t_cal) * 1e3))
    est = min(ests)
    reps = int(max_over_ranks(world, float(repeats_for(args.min_timed_s, est)), device=dev))
    barrier(world)
    rep_ms, call_ms = [], []
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(world)
        l0 = km.launch_count()
        t0 = time.perf_counter()
        for _ in range(reps):
            a, b = one_fit(args.steps)
            rep_ms.append(a)
            call_ms.append(b)
        torch.cuda.synchronize()
        timed_s = time.perf_counter() - t0
        launches = km.launch_count() - l0
    barrier(world)
    ms = _median(rep_ms)                 # device time of exactly `steps` iterations
    ms_max = max_over_ranks(world, ms, device=dev)
    ms_call_max = max_over_ranks(world, _median(call_ms), device=dev)
    res = None
    # Phase split from one more fit of the same problem right after the timed
    # region (the device is still at its loaded clock): events between the
    # assignment and the update stop those kernels from overlapping their
    # launches, so it is kept apart from `value`.
    phase = km.fit_profile(X, C0, args.steps)["phase_ms"] if not dp else None
    # The same fit replayed as a CUDA graph (km_fit_graph_*): device time of
    # the whole call, comparable with value_call.
    graph_ms = graph_call_ms(km, X, C0, args.steps) if not dp and rank == 0 else None
    if rank == 0:
        pk, pk_kind = peaks()
        value = job_rate(args.steps, world, ms_max)
        res = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": workload_config(wl, world, parallelism),
            "repeats": reps, "timed_region_s": round(timed_s, 3),
            "ms_per_step_each_repeat": [round(v / args.steps, 4) for v in rep_ms[:64]],
            "value_call": round(job_rate(args.steps, world, ms_call_max), 3),
            "value_graph_call": round(job_rate(args.steps, 1, graph_ms), 3) if graph_ms else None,
            "ms_call": round(ms_call_max, 4),
            "gpu_launches": int(launches),
            "gpu_launches_per_repeat": int(launches) // reps,
            "clocks": clk.summary(),
        }
        if phase is not None:
            assign_ms = float(phase[:, 0].mean())
            update_ms = float(phase[:, 1].mean())
            af, ub = assign_flops(wl), update_bytes(wl)
            a_tf = af / (assign_ms * 1e-3) / 1e12
            u_gbs = ub / (update_ms * 1e-3) / 1e9
            # A kernel timed inside a long run (a timed region of a second or
            # more) runs at the power-capped clock: its tensor peak is the
            # sustained cuBLAS figure; a short burst compares with the burst one.
            long_run = timed_s >= 1.0
            tpk = pk["bf16_tflops_sustained"] if long_run else pk["bf16_tflops"]
            res["phases"] = {"assign_ms": round(assign_ms, 4), "assign_tflops": round(a_tf, 2),
                             "assign_frac_of_bf16_burst": round(a_tf / pk["bf16_tflops"], 4),
                             "assign_frac_of_bf16_sustained": round(a_tf / pk["bf16_tflops_sustained"], 4),
                             "update_ms": round(update_ms, 4), "update_gbs": round(u_gbs, 1),
                             "update_frac_of_hbm": round(u_gbs / pk["hbm_gbs"], 4),
                             "update_algorithmic_bytes": ub, "assign_algorithmic_flops": af}
            if assign_ms >= update_ms:
                res["roofline"] = {
                    "bound": "tensor", "kernel": "k_assign", "achieved": round(a_tf, 2), "peak": tpk,
                    "unit": "TFLOP/s", "frac": round(a_tf / tpk, 4), "frac_of_burst": round(a_tf / pk["bf16_tflops"], 4),
                    "peak_kind": f"{pk_kind} bf16 {'sustained' if long_run else 'burst'}",
                    "traffic": recorded_traffic("k_assign", wl.name), "algorithmic_per_launch": af}
            else:
                res["roofline"] = {
                    "bound": "hbm", "kernel": "update", "achieved": round(u_gbs, 1), "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": round(u_gbs / pk["hbm_gbs"], 4), "peak_kind": f"{pk_kind} copy",
                    "traffic": recorded_traffic("update", wl.name), "algorithmic_per_launch": ub}
        else:
            res["phases"] = None
            res["roofline"] = {"bound": "tensor", "kernel": "k_assign", "achieved": None, "peak": None,
                               "unit": "TFLOP/s", "frac": None, "traffic": None,
                               "note": "data-parallel run: per-phase split not taken (the exchange sits between)"}
        if world == 1 and args.tile_sweep:
            res["tile_sweep"] = tile_sweep(wl, X, C0, km)
        if world == 1 and args.ablation and wl.B == 1:
            res["ablation"] = ablation(wl, X, C0, km, res["phases"]["assign_ms"], res["phases"]["update_ms"])
        if world == 1 and not args.no_e2e:
            res["e2e"] = e2e(args, wl, X, C0, km)
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl, X, C0, args.cpu_seconds)
    return res


def graph_call_ms(km, X, C0, steps, budget_s=0.3):
    """Median device time of one launch of the fit captured as a CUDA graph
    (events around each launch), over launches worth about budget_s."""
    g = km.FitGraph(X, C0, steps, want_idx=False)
    try:
        for _ in range(3):
            g.launch()
        torch.cuda.synchronize()
        first = _event_ms(g.launch, reps=1)
        n = max(5, min(200, int(budget_s * 1e3 / max(first, 1e-3))))
        return _event_ms(g.launch, reps=n)
    finally:
        g.close()


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
    """The out-of-core workloads: X lives in pinned host memory and every
    iteration streams it to the device in chunks (copies overlapped with the
    assignment and update of the previous chunk).  The step is one Lloyd
    iteration over all N points, through km_fit_host (ooc_268m_k4096) or,
    for a set never held whole (ooc_1b_k4096: 2^30 rows, row i = pool row
    i mod 2^28), through km_fit_source with a source that points into the
    pool.  The host link, not a kernel, bounds these, so the roofline
    reports host->device bytes against the pinned copy bandwidth measured
    here."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    chunk = 16 << 20
    pw = pool_workload(wl)
    Xh = torch.empty((pw.N, wl.D), dtype=wl.torch_dtype, pin_memory=True)
    make_points(pw, seed=args.seed, device=dev, out=Xh)
    sel = init_rows(wl, args.seed, dev).cpu()
    C0 = Xh[sel].to(dev).contiguous()
    torch.cuda.synchronize()
    link = h2d_link_gbs(Xh[:chunk], dev)
    P = pw.N

    def source(row0, rows, slot):
        r = row0 % P
        return Xh[r:r + rows]

    def fit(iters):
        if wl.pool_rows:
            return km.fit_source(source, wl.N, C0, iters, chunk)
        return km.fit_host(Xh, C0, iters, chunk)

    fit(args.warmup)
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        l0 = km.launch_count()
        t0 = time.perf_counter()
        r = fit(args.steps)
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
        "config": workload_config(wl, 1, "single"),
        "timed_region_s": round(dt, 3),
        "roofline": {"bound": "h2d", "kernel": "chunk stream", "achieved": round(achieved, 1),
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
        res["cpu_baseline"] = cpu_baseline(wl, Xh, C0, args.cpu_seconds)
    return res


def e2e(args, wl, X, C0, km):
    """Same metric through the public API with host buffers: every iteration
    streams X from pinned host memory (chunks overlapped with compute), and
    the objective history and final centroids are read back to the host."""
    if wl.B > 1:
        return e2e_batched(args, wl, X, C0, km)
    Xh = X.reshape(-1, wl.D).cpu().pin_memory()
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


def e2e_batched(args, wl, X, C0, km):
    """Batched problems (km_fit_host streams one instance): every step copies
    all instances' points and initial centroids from pinned host memory,
    runs one Lloyd iteration with km_fit, and reads the new centroids and
    the objective back; wall clock around the steps."""
    Xh, Ch = X.cpu().pin_memory(), C0.cpu().pin_memory()
    Xd, Cd = torch.empty_like(X), torch.empty_like(C0)
    C_host = torch.empty((wl.B, wl.K, wl.D), dtype=torch.float32).pin_memory()
    obj_host = torch.empty((wl.B, 1), dtype=torch.float64).pin_memory()

    def step():
        Xd.copy_(Xh, non_blocking=True)
        Cd.copy_(Ch, non_blocking=True)
        r = km.fit(Xd, Cd, 1, want_idx=False)
        C_host.copy_(r["C"], non_blocking=True)
        obj_host.copy_(r["objective"], non_blocking=True)

    step()  # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    h2d = X.numel() * X.element_size() + C0.numel() * C0.element_size()
    d2h = C_host.numel() * 4 + obj_host.numel() * 8
    return {"value": round(args.steps / dt, 3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
            "how": "per step: all instances' X and C0 copied from pinned host memory, one km_fit iteration, "
                   "centroids and objective read back; wall clock around the steps"}


def run_reference(args, world, rank):
    """The oracle (plain float64 C on the host cores), as it stands, on a
    bounded seeded row sample of the same workload: the same X and C0 as the
    GPU arm (drawn with the CUDA generator when a GPU is present), the sample
    sized so that the W warm-up and K timed iterations together take about
    --ref-seconds of host work.  Rank 0 alone runs it."""
    if rank != 0:
        return None
    import oracle
    wl = WORKLOADS[args.workload]
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    if wl.host_resident:
        # rows are iid: the first rows of the host-resident set (of its pool)
        # are a sample of it
        base = pool_workload(wl).with_(N=min(pool_workload(wl).N, 1 << 22), host_resident=False)
        X, C0 = make_inputs(base, args.seed, gen_dev)
    else:
        X, C0 = make_inputs(wl if wl.B == 1 else wl.with_(B=1), args.seed, gen_dev)
    total = args.steps + args.warmup
    Xs, Cs = oracle_rows(wl, X, C0, args.ref_seconds, total)
    n = Xs.shape[0]
    oracle.fit(Xs, Cs, args.warmup, mirror=wl.dtype)
    t0 = time.perf_counter()
    oracle.fit(Xs, Cs, args.steps, mirror=wl.dtype)
    dt = time.perf_counter() - t0
    per_iter_full = dt / args.steps * (wl.N * wl.B / n)
    value = 1.0 / per_iter_full
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_iter_full * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(wl, world, "single" if world == 1 else f"dp{world}"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{n} of {wl.N * wl.B} points (seeded uniform sample of the same X, drawn on "
                                       f"{gen_dev}), all K={wl.K} centroids, {args.warmup} + {args.steps} iterations, "
                                       f"{dt:.1f} s timed; rate scaled linearly to the full point count"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parallelism", default="dp", choices=["dp", "replicas"],
                    help="with several ranks: shard one problem by rows (dp) or run independent replicas")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--dist-backend", default="nccl", choices=["nccl", "gloo"],
                    help="gloo only for a single-GPU smoke run of the multi-rank path (with --same-device)")
    ap.add_argument("--same-device", action="store_true",
                    help="every rank on cuda:0 (smoke run of the multi-rank path on one GPU)")
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="repeat the K-step fit until the timed region lasts this long")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="host work of the CPU-baseline sample")
    ap.add_argument("--ref-seconds", type=float, default=120.0, help="host work of the reference arm")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tile-sweep", action="store_true",
                    help="also time every assignment tiling that fits against the static choice")
    ap.add_argument("--ablation", action="store_true",
                    help="also time the materialised-distance and atomic-scatter baselines")
    ap.add_argument("--record-traffic", metavar="CSV",
                    help="store the DRAM traffic of --kernel from an ncu raw CSV export and exit")
    ap.add_argument("--kernel", default="k_assign", choices=sorted(KERNEL_SOURCES))
    ap.add_argument("--traffic-scale", type=float, default=1.0,
                    help="full-size units / captured units, for a capture of a smaller case")
    ap.add_argument("--traffic-command", default="", help="the ncu command the CSV came from")
    args = ap.parse_args()
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, args.kernel, args.workload, args.traffic_scale,
                                        args.traffic_command)))
        return
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, world, rank)
    else:
        world, rank, local = dist_setup(args.gpus, args.dist_backend, args.same_device)
        res = run_ours(args, world, rank, local)
        if world > 1:
            torch.distributed.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
