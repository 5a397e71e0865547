#!/usr/bin/env python
"""Benchmark of the reduced cross-entropy loss, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sasrec]

One step = the whole path on one batch: bucketing + sort (rece_bucketize_sort), chunk
scores + top-k + loss (rece_loss_fwd) and gradients (rece_loss_bwd), with fresh random
vectors B every step.  Inputs are synthetic (seeded, shaped like the RECE paper's
SASRec workloads) and resident in HBM; L2 is flushed (a 256 MiB write) between timed
steps because the inputs fit in L2.  Multi-GPU: every rank runs the whole path on its own
batch against its own copy of the catalogue (weak scaling, no collective on the data
path); the time is the max over ranks.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle instead (a
deliberately slow baseline, rank 0 only).
"""
import argparse
import ctypes
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

METRIC = "rows/sec RECE loss fwd+bwd (1×B200), % roofline, peak HBM vs full CE"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="sasrec")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-memory", action="store_true")
    ap.add_argument("--no-allreduce-dy", action="store_true",
                    help="N > 1: run independent replicas, without summing dY across ranks")
    ap.add_argument("--no-baselines", action="store_true",
                    help="skip timing the sampled CE- / BCE+ comparison ops")
    ap.add_argument("--flags", type=int, default=0, help="rece_config_t.flags")
    return ap.parse_args()


def workload_desc(w):
    return (f"{w.name}: N={w.N} (rows), d={w.d}, C={w.C}, {w.dtype}, n_b={w.n_b}, n_c={w.n_c}, "
            f"n_ec={w.n_ec}, n_r={w.n_r}, k={w.k}, targets "
            + (f"Zipf({w.target_alpha})" if w.target_alpha else "uniform"))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"),
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


# ------------------------------------------------------------------ algorithmic work
def chunk_start(c, M, n_c):
    return (c * M + n_c - 1) // n_c


def pairs_per_round(w):
    """Sum over chunks of (rows in chunk) x (items in its window)."""
    tot = 0
    for c in range(w.n_c):
        rows = chunk_start(c + 1, w.N, w.n_c) - chunk_start(c, w.N, w.n_c)
        lo, hi = max(0, c - w.n_ec), min(w.n_c, c + w.n_ec + 1)
        tot += rows * (chunk_start(hi, w.C, w.n_c) - chunk_start(lo, w.C, w.n_c))
    return tot


def stage_work(w, paths=0):
    """Algorithmic (flops, bytes) of every stage, per step (one launch sequence)."""
    from reduced_cross_entropy_b200 import _lib
    e = 2 if w.dtype == "bf16" else 4
    N, C, d, nb, nr, k = w.N, w.C, w.d, w.n_b, w.n_r, w.k
    if paths & _lib.PATH_ALL_NEGATIVES:
        # Algorithm 1 as printed: every window pair scored in the forward, and in the
        # backward scored again and multiplied twice (dX = P Y, dY = P^T X); the positives
        # through the pair backward
        pr = pairs_per_round(w) * nr
        return {
            "bucketize": (2 * (N + C) * nb * d * nr, nr * (N + C) * (d * e + 4)),
            "sort": (0, nr * (N + C) * (16 + 2 * d * e)),
            "select": (2 * d * pr, nr * (N + C) * d * e + 8 * nr * N),
            "merge_loss": (0, 8 * nr * N + 2 * N * d * e + 8 * N),
            "mean": (0, 4 * N),
            "bwd_rows": (4 * d * pr + 2 * N * d, nr * (N + C) * d * e + 2 * N * d * 4),
            "bwd_sort": (0, 0),
            "bwd_items": (4 * d * pr, nr * (N + C) * d * e + 2 * C * d * 4),
        }
    # Step 6 charges what the scope table does: F = 4 N (k+1) d, B = (N+C) d e + 8 N k +
    # (N+C) d 4 -- X and Y read once, dX and dY written once -- split between the dX
    # stage (Y, the coefficients' inputs, dX) and the dY stage (X, dY); re-reading a
    # gathered row and the pair sort are the implementation's cost, not charged.
    tc = paths & _lib.PATH_TENSOR_CORES
    return {
        "bucketize": (2 * (N + C) * nb * d * nr, nr * (N + C) * (d * e + 4)),
        "sort": (0, nr * (N + C) * (16 + (2 * d * e if tc else 0))),
        "select": (2 * d * pairs_per_round(w) * nr, nr * (N + C) * d * e + nr * N * k * 8),
        "merge_loss": (0, nr * N * k * 8 + N * k * 4 + 8 * N),
        "mean": (0, 4 * N),
        "bwd_rows": (2 * N * (k + 1) * d, C * d * e + 8 * N * k + N * d * 4),
        "bwd_sort": (0, 0),
        "bwd_items": (2 * N * (k + 1) * d, N * d * e + C * d * 4),
    }


def stage_bound(stage, paths):
    """The roofline a stage is held to, given the plan's kernels (rece_plan_paths)."""
    from reduced_cross_entropy_b200 import _lib
    if stage in ("bucketize", "select"):
        return "tensor" if paths & _lib.PATH_TENSOR_CORES else "alu"
    if stage in ("bwd_rows", "bwd_items") and paths & _lib.PATH_ALL_NEGATIVES:
        return "tensor"
    if stage == "bwd_rows" and paths & _lib.PATH_DX_TENSORS:
        return "tensor"
    return "hbm"  # (the pair sort has no algorithmic work: its fraction reads 0)


KERNEL_SOURCES = {  # the pair sort's pass geometry is decided in rece_abi.cu
    "bucketize": ["bucketize.cu"], "sort": ["sort.cu"], "select": ["select.cu"],
    "merge_loss": ["loss.cu"], "mean": ["loss.cu"], "bwd_rows": ["backward.cu"],
    "bwd_sort": ["sort.cu", "rece_abi.cu"], "bwd_items": ["backward.cu"],
}


def kernel_sources(stage, paths):
    from reduced_cross_entropy_b200 import _lib
    src = dict(KERNEL_SOURCES)
    if paths & _lib.PATH_TENSOR_CORES:
        src.update(bucketize=["bucketize_tc.cu", "sm100.cuh"], sort=["sort.cu", "permute.cu"],
                   select=["select_tc.cu", "sm100.cuh", "tc_bins.cuh"],
                   merge_loss=["merge_tc.cu"])
    if paths & _lib.PATH_STORED_SCORES:
        src["select"] = ["scores_tc.cu", "sm100.cuh", "tc_bins.cuh"]
    if paths & _lib.PATH_DX_TENSORS:
        src["bwd_rows"] = ["backward.cu", "bwd_tc.cu", "sm100.cuh", "tc_common.cu"]
    if paths & _lib.PATH_DY_TENSORS:  # the positives' pair backward, then the band products
        src.update(bwd_sort=["backward.cu", "sort.cu", "rece_abi.cu"],
                   bwd_items=["bwd_tc.cu", "sm100.cuh"])
    if paths & _lib.PATH_ALL_NEGATIVES:
        src.update(select=["window_tc.cu", "window.cu", "sm100.cuh"],
                   merge_loss=["window.cu"],
                   bwd_rows=["backward.cu", "window_tc.cu", "tc_common.cu"],
                   bwd_sort=["sort.cu", "rece_abi.cu"], bwd_items=["window_tc.cu"])
    return src[stage]


def source_hash(stage, paths):
    h = hashlib.sha256()
    for f in kernel_sources(stage, paths):
        h.update(open(os.path.join(ROOT, "reduced_cross_entropy_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(stage, workload, paths):
    """DRAM bytes per step of this stage (all its launches) from a committed ncu capture,
    if the kernel sources are unchanged since (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{stage}@{workload}@paths{paths}")
    if not d or d.get("source_sha") != source_hash(stage, paths):
        return None
    return d.get("dram_bytes_per_step")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle timing
def oracle_step_seconds(w, X, Y, t, B, rows=256, bucket_frac=16, all_negatives=False):
    """Estimated seconds of one whole step of the CPU oracle, from a bounded sample:
    bucketing of every bucket_frac-th row of X and Y (scaled up), the full stable sorts,
    and selection + loss + gradient of `rows` rows (scaled by N / rows)."""
    import oracle
    n_r = w.n_r
    t0 = time.perf_counter()
    for r in range(n_r):
        oracle.bucketize(X[::bucket_frac], B[r])
        oracle.bucketize(Y[::bucket_frac], B[r])
    t_bucket = (time.perf_counter() - t0) * bucket_frac
    # valid orders for the sampled rows come from a full (untimed) bucketing, once
    if not hasattr(oracle_step_seconds, "_perm"):
        bx = np.stack([oracle.bucketize(X, B[r]) for r in range(n_r)])
        by = np.stack([oracle.bucketize(Y, B[r]) for r in range(n_r)])
        oracle_step_seconds._perm = (bx, by)
    bx, by = oracle_step_seconds._perm
    t0 = time.perf_counter()
    px = np.stack([oracle.stable_argsort(bx[r]) for r in range(n_r)])
    py = np.stack([oracle.stable_argsort(by[r]) for r in range(n_r)])
    t_sort = time.perf_counter() - t0
    sample = np.linspace(0, w.N - 1, rows).astype(np.int64)
    t0 = time.perf_counter()
    if all_negatives:  # Algorithm 1 as printed: every window item a negative
        _, _, lse = oracle.window_loss(X, Y, t, px, py, w.n_c, w.n_ec, rows=sample)
        oracle.window_grad(X, Y, t, px, py, w.n_c, w.n_ec, lse, 1.0, rows=sample)
        return t_bucket + t_sort + (time.perf_counter() - t0) * w.N / rows
    sel, _, _ = oracle.select(X, Y, t, px, py, w.n_c, w.n_ec, w.k, rows=sample)
    _, _, lse = oracle.rece_loss(X[sample], Y, t[sample], sel)
    oracle.rece_grad(X[sample], Y, t[sample], sel, lse, 1.0)
    t_rows = (time.perf_counter() - t0) * w.N / rows
    return t_bucket + t_sort + t_rows


def oracle_sample_desc(rows, bucket_frac):
    return (f"bucketing of every {bucket_frac}th row of X and Y (x{bucket_frac}), full stable "
            f"sorts, selection+loss+gradient of {rows} evenly spaced rows (x N/{rows})")


def run_reference(args):
    rank, _, _ = dist_env()
    if rank != 0:  # the oracle arm runs on rank 0 alone; other ranks exit without work
        return
    import oracle
    from reduced_cross_entropy_b200 import synth
    w = synth.WORKLOADS[args.workload]
    X, Y, t = synth.make_inputs(w, seed=0)
    B = synth.projections(0, 0, w.n_r, w.n_b, w.d, w.dtype)
    rows, frac = 128, 32
    alln = bool(getattr(args, "flags", 0) & 0x2)  # RECE_FLAG_ALL_NEGATIVES: Algorithm 1 as printed
    for _ in range(args.warmup):
        oracle_step_seconds(w, X, Y, t, B, rows, frac, all_negatives=alln)
    secs = [oracle_step_seconds(w, X, Y, t, B, rows, frac, all_negatives=alln)
            for _ in range(args.steps)]
    total = sum(secs)
    value = w.N * args.steps / total
    cores = oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(w)},
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": cores, "kind": "oracle",
                             "sample": oracle_sample_desc(rows, frac)},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ranks
def dist_env():
    """(rank, local_rank, world) from the launcher's environment (torchrun sets them)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(x, device=None):
    """The largest x over the ranks of the default process group (x itself with no group).
    Every rank must call it, in the same order.  device: where the reduction tensor
    lives (the rank's GPU under NCCL, the CPU under gloo)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_dy(dY):
    """Data-parallel replicas share the catalogue Y: the one exchange of a training step
    is the sum of the ranks' dY (NCCL over NVLink under torchrun; any backend of the
    default group).  Every rank calls it once per step, in the same place."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dY, op=dist.ReduceOp.SUM)


def job_throughput(world, rows_per_step, steps, total_ms):
    """Whole-job rows/s: every rank processes rows_per_step rows per step (weak scaling),
    timed by the slowest rank's total_ms over `steps` steps."""
    return world * rows_per_step * steps / (total_ms / 1000.0)


# ------------------------------------------------------------------ GPU arm
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from reduced_cross_entropy_b200 import _lib, ops, synth

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    exchange = world > 1 and not args.no_allreduce_dy

    L = _lib.lib()
    w = synth.WORKLOADS[args.workload]
    X, Y, t = synth.make_inputs(w, seed=rank)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype,
                    flags=args.flags)
    Xd = torch.from_numpy(X).to(dev).to(tdt)
    Yd = torch.from_numpy(Y).to(dev).to(tdt)
    td = torch.from_numpy(t).to(dev)
    n_steps = args.warmup + args.steps
    Bs = [torch.from_numpy(synth.projections(0, s, w.n_r, w.n_b, w.d, w.dtype)).to(dev).to(tdt)
          for s in range(n_steps)]
    ws = plan.workspace(dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    sel = torch.empty(w.N, w.k, dtype=torch.int32, device=dev)
    lse = torch.empty(w.N, dtype=torch.float32, device=dev)
    logits = torch.empty(w.N, w.k + 1, dtype=torch.float32, device=dev)
    dloss = torch.ones(1, dtype=torch.float32, device=dev)
    dX = torch.empty(w.N, w.d, dtype=torch.float32, device=dev)
    dY = torch.empty(w.C, w.d, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    vp = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
    nbytes = ctypes.c_size_t(ws.numel())

    def step(Bt, Xc=None, Yc=None, tc=None):
        Xc = Xd if Xc is None else Xc
        Yc = Yd if Yc is None else Yc
        tc = td if tc is None else tc
        _lib.check(L.rece_bucketize_sort(plan._h, vp(Bt), vp(Xc), vp(Yc), vp(ws), nbytes, sp),
                   "bucketize_sort")
        _lib.check(L.rece_loss_fwd(plan._h, vp(Xc), vp(Yc), vp(tc), vp(ws), nbytes, vp(loss),
                                   None, vp(sel), vp(lse), vp(logits), sp), "loss_fwd")
        _lib.check(L.rece_loss_bwd(plan._h, vp(Xc), vp(Yc), vp(tc), vp(sel), vp(lse),
                                   vp(logits), vp(dloss), vp(ws), nbytes, vp(dX), vp(dY), sp),
                   "loss_bwd")
        if exchange:
            allreduce_dy(dY)

    for s in range(args.warmup):
        flush.zero_()
        step(Bs[s])
    torch.cuda.synchronize(dev)
    # status area: flags (a bad target or a timed-out wait fails the run; the tensor-core
    # selection may flag rows it cannot certify exact) and the count of such rows
    status_words = ws[:16].view(torch.int32).cpu().tolist()
    assert status_words[0] & ~_lib.DEVICE_INEXACT == 0, f"device status {status_words[0]:#x}"
    inexact_rows, overflow_rows = int(status_words[1]), int(status_words[2])
    spilled_rows = int(status_words[3])

    # timed region: K steps, each bracketed by events; per-stage events recorded by the
    # library on the same stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    n_st = len(_lib.STAGES)
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n_st)]
           for _ in range(args.steps)]
    for row in sev:  # torch creates the CUDA event at its first record
        for e in row:
            e.record(stream)
    sev_h = [(ctypes.c_void_p * (2 * n_st))(*[ctypes.c_void_p(e.cuda_event) for e in row])
             for row in sev]
    launches0 = L.rece_kernel_launch_count()
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        for s in range(args.steps):
            flush.zero_()
            _lib.check(L.rece_plan_set_stage_events(plan._h, sev_h[s]), "stage events")
            ev[s][0].record(stream)
            step(Bs[args.warmup + s])
            ev[s][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    launches = L.rece_kernel_launch_count() - launches0
    L.rece_plan_set_stage_events(plan._h, None)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), dev)
    stage_ms = {name: statistics.mean(sev[s][2 * i].elapsed_time(sev[s][2 * i + 1])
                                      for s in range(args.steps))
                for i, name in enumerate(_lib.STAGES)}
    value = job_throughput(world, w.N, args.steps, total_ms)

    # roofline of every stage, the dominant one reported as the line's roofline
    peaks = load_peaks()
    paths = plan.paths
    work = stage_work(w, paths)

    def stage_roofline(name):
        bound = stage_bound(name, paths)
        flops, bytes_ = work[name]
        sec = max(stage_ms[name], 1e-9) / 1000.0
        if bound == "hbm":
            achieved, peak, unit = bytes_ / sec / 1e9, peaks["hbm_gbs"], "GB/s"
        elif bound == "tensor":
            achieved, peak, unit = flops / sec / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        else:  # fp32 FMA on the CUDA cores: 148 SMs x 128 lanes x 2 flop x max SM clock
            achieved, peak, unit = (flops / sec / 1e12,
                                    148 * 128 * 2 * peaks["sm_max_mhz"] / 1e6, "TFLOP/s")
        return {"bound": bound, "kernel": name, "achieved": achieved, "peak": peak,
                "unit": unit, "frac": achieved / peak,
                "peak_source": peaks["source"] if bound != "alu" else
                "derived: 148 SM x 128 FP32 lanes x 2 x sm_max_mhz",
                "traffic": recorded_traffic(name, w.name, paths),
                "algorithmic_bytes": bytes_, "algorithmic_flops": flops}

    dom = max(stage_ms, key=stage_ms.get)
    roofline = stage_roofline(dom)
    stage_fracs = {name: round(stage_roofline(name)["frac"], 4) for name in stage_ms}

    # end to end: every step's inputs copied in from pinned host memory and its loss
    # copied out, through the same C-ABI calls.  Step s+1's copies (a copy stream, two
    # device input sets) overlap step s's compute, as a training input pipeline does; the
    # L2 flush stays in the timeline; one pair of events spans all timed steps.
    Xh = torch.from_numpy(X).to(tdt).pin_memory()
    Yh = torch.from_numpy(Y).to(tdt).pin_memory()
    th = torch.from_numpy(t).pin_memory()
    Bh = [b.cpu().pin_memory() for b in Bs]
    loss_h = torch.empty(n_steps, dtype=torch.float32).pin_memory()
    h2d = Xh.numel() * Xh.element_size() + Yh.numel() * Yh.element_size() + th.numel() * 4 \
        + Bh[0].numel() * Bh[0].element_size()
    sets = [(Xd, Yd, td, torch.empty_like(Bs[0])),
            (torch.empty_like(Xd), torch.empty_like(Yd), torch.empty_like(td),
             torch.empty_like(Bs[0]))]
    cstream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def issue_copy(s, j):
        k = s % 2
        with torch.cuda.stream(cstream):
            if j >= 2:  # the set's previous step has finished with it
                cstream.wait_event(consumed[k])
            for dst, src in zip(sets[k], (Xh, Yh, th, Bh[s])):
                dst.copy_(src, non_blocking=True)
            copied[k].record(cstream)

    def e2e_run(first, count):
        torch.cuda.synchronize(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(cstream)
        issue_copy(first, 0)
        for j in range(count):
            s = first + j
            if j + 1 < count:
                issue_copy(s + 1, j + 1)
            k = s % 2
            stream.wait_event(copied[k])
            flush.zero_()
            Xc, Yc, tc, Bc = sets[k]
            step(Bc, Xc, Yc, tc)
            consumed[k].record(stream)
            loss_h[s].copy_(loss[0], non_blocking=True)
        t1.record(stream)
        t1.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(0, args.warmup)
    barrier()
    e2e_ms = [e2e_run(args.warmup, args.steps)]
    assert np.all(np.isfinite(loss_h.numpy())), "non-finite loss"
    e2e_total = max_over_ranks(sum(e2e_ms), dev)
    e2e = {"value": job_throughput(world, w.N, args.steps, e2e_total), "unit": "rows/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 4}

    line = {"metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": workload_desc(w), "inexact_rows_per_step": inexact_rows,
                       "overflowed_rows_per_step": overflow_rows,
                       "merge_spilled_rows_per_step": spilled_rows,
                       "l2": "flushed between timed steps (256 MiB write)",
                       "parallelism": f"dp{world}",
                       "exchange": ("all-reduce of dY [C x d] fp32 every step (NCCL)"
                                    if exchange else "none"),
                       "scores": ("tcgen05" + (", stored" if paths & _lib.PATH_STORED_SCORES
                                                 else ", recomputed per pass")
                                  if paths & _lib.PATH_TENSOR_CORES else "fmaf CUDA cores"),
                       "dX": ("tcgen05 band products" +
                              (", rounds in one launch, parts summed in order"
                               if paths & _lib.PATH_DX_PARTS else "")
                              if paths & _lib.PATH_DX_TENSORS else "gathered rows"),
                       "negatives": ("every window item (Algorithm 1 as printed), window "
                                     "sums and gradients on tcgen05"
                                     if paths & _lib.PATH_ALL_NEGATIVES
                                     else f"top-{w.k} per row")},
            "roofline": roofline, "stages_ms": stage_ms, "stages_roofline_frac": stage_fracs,
            "e2e": e2e, "gpu_launches": int(launches),
            "clocks": clk.summary()}

    if rank == 0 and world == 1 and not args.no_memory:
        line["peak_hbm"] = measure_memory(torch, ops, plan, w, Xd, Yd, td, Bs[0], dev)
    if rank == 0 and world == 1 and not args.no_baselines:
        line["baselines"] = measure_baselines(torch, ops, w, Xd, Yd, td, flush, dev,
                                              load_peaks())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        rows, frac = 256, 16
        secs = oracle_step_seconds(w, X, Y, t, synth.projections(0, 0, w.n_r, w.n_b, w.d,
                                                                   w.dtype), rows, frac,
                                   all_negatives=bool(paths & _lib.PATH_ALL_NEGATIVES))
        line["cpu_baseline"] = {"value": w.N / secs, "unit": "rows/s",
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": oracle_sample_desc(rows, frac)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_baselines(torch, ops, w, Xd, Yd, td, flush, dev, peaks, reps=10, warm=3):
    """The pages' sampled comparison points (RECE section 2: CE- eq. 2, BCE+ eq. 1) on the
    same resident inputs, n = k uniform negatives per row (as many as RECE keeps):
    fwd+bwd rows/s (L2 flushed between steps, CUDA events), and the forward's gather
    rate: its algorithmic bytes are the N (n+1) catalogue rows it reads, x, and the
    logits it writes."""
    from reduced_cross_entropy_b200 import synth
    n = w.k
    neg = torch.from_numpy(synth.uniform_negatives(1, w.N, w.C, n)).to(dev)
    dl = torch.ones(1, dtype=torch.float32, device=dev)
    e = 2 if w.dtype == "bf16" else 4
    fwd_bytes = w.N * (n + 1) * w.d * e + w.N * w.d * e + w.N * (n + 1) * 4
    out = {"negatives_per_row": n, "sampling": "uniform over [0, C), with replacement"}
    stream = torch.cuda.current_stream(dev)
    for kind in ("ce_minus", "bce_plus"):
        ws = torch.empty(ops.sampled_workspace_bytes(kind, w.N, w.C, w.d, n, w.dtype),
                         dtype=torch.uint8, device=dev)
        fw, tot = [], []
        for r in range(warm + reps):
            flush.zero_()
            a, m, b = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record(stream)
            _, _, lg, lse, _ = ops.sampled_fwd(kind, Xd, Yd, td, neg, ws)
            m.record(stream)
            ops.sampled_bwd(kind, Xd, Yd, td, neg, lse, dl, ws, logits=lg)
            b.record(stream)
            b.synchronize()
            if r >= warm:
                fw.append(a.elapsed_time(m))
                tot.append(a.elapsed_time(b))
        assert ops.device_status(ws) == 0
        ms, fms = statistics.median(tot), statistics.median(fw)
        gbs = fwd_bytes / (fms / 1e3) / 1e9
        out[kind] = {"rows_per_s": w.N / (ms / 1e3), "ms_fwd_bwd": ms, "ms_fwd": fms,
                     "fwd_gather_gbs": gbs, "fwd_frac_of_hbm": gbs / peaks["hbm_gbs"]}
    return out


def measure_memory(torch, ops, plan, w, Xd, Yd, td, B, dev):
    """Peak HBM of one RECE fwd+bwd vs the fused exact full CE and the materialised
    full CE (logits + their gradient in fp32), all from the same resident inputs."""
    out = {}
    base = torch.cuda.memory_allocated(dev)

    def peak(fn):
        torch.cuda.synchronize(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        fn()
        torch.cuda.synchronize(dev)
        return torch.cuda.max_memory_allocated(dev) - base

    def rece():
        ws = plan.workspace(dev)
        ops.bucketize_sort(plan, B, Xd, Yd, ws)
        _, _, s, l, lg = ops.loss_fwd(plan, Xd, Yd, td, ws, want_row_loss=False)
        ops.loss_bwd(plan, Xd, Yd, td, s, l, torch.ones(1, device=dev), ws, logits=lg)

    def fused():
        _, _, l, ws = ops.full_ce_fwd(Xd, Yd, td)
        ops.full_ce_bwd(Xd, Yd, td, l, torch.ones(1, device=dev), ws)

    out["rece_bytes"] = peak(rece)
    # the fused exact op runs on the CUDA cores: past ~3e13 flops (minutes) it is skipped
    if 6.0 * w.N * w.C * w.d <= 3e13:
        out["full_ce_fused_bytes"] = peak(fused)
    else:
        out["full_ce_fused_bytes"] = None
        out["full_ce_fused_note"] = "skipped: 6 N C d flops on the CUDA cores would take minutes"
    mat = 8 * w.N * w.C
    out["full_ce_materialised_bytes_computed"] = mat
    free = torch.cuda.mem_get_info(dev)[0]
    if 3 * mat < free:
        def materialised():
            Xr = Xd.float().requires_grad_()
            Yr = Yd.float().requires_grad_()
            torch.nn.functional.cross_entropy(Xr @ Yr.T, td.long()).backward()
        out["full_ce_materialised_bytes_measured"] = peak(materialised)
    ref = out.get("full_ce_materialised_bytes_measured", mat)
    out["ratio_vs_materialised"] = ref / max(out["rece_bytes"], 1)
    if out["full_ce_fused_bytes"] is not None:
        out["ratio_vs_fused"] = out["full_ce_fused_bytes"] / max(out["rece_bytes"], 1)
    # the pages' memory model of Algorithm 1 (every chunk's logits stored) at this
    # workload's alpha_bc = n_b / n_c, and the bucket count it calls optimal
    a = w.n_b / w.n_c
    nb, nc = ops.optimal_buckets(w.N, w.C, w.n_ec, a)
    el = ops.memory_model_elements(w.N, w.C, w.n_ec, w.n_r, a)
    out["pages_memory_model"] = {"alpha_bc": a, "n_b_star": nb, "n_c_star": nc,
                                 "logit_elements": el, "bytes_fp32": 4 * el,
                                 "rece_bytes_over_model": out["rece_bytes"] / (4 * el)}
    out["note"] = "bytes above the resident inputs; torch.cuda.max_memory_allocated"
    return out


if __name__ == "__main__":
    main()
