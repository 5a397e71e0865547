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
    ap.add_argument("--workload", default="very_large",
                    help="the headline workload (synth.WORKLOADS)")
    ap.add_argument("--also", default="large,sasrec",
                    help="one GPU: more workloads measured in the same run, reported under "
                         "'workloads' (comma-separated; empty for none)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-memory", action="store_true")
    ap.add_argument("--no-allreduce-dy", action="store_true",
                    help="N > 1: run independent replicas, without summing dY across ranks")
    ap.add_argument("--no-baselines", action="store_true",
                    help="skip timing the sampled CE- / BCE+ comparison ops")
    ap.add_argument("--flags", type=int, default=0, help="rece_config_t.flags")
    ap.add_argument("--slice", type=int, default=1,
                    help="run a proportional 1/F slice of the workload (N, C and n_c divided "
                         "by F: the same chunks and windows), e.g. for profiler captures")
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
    if paths & _lib.PATH_ALL_NEGATIVES and paths & _lib.PATH_WINDOW_FMA:
        return "alu" if stage in ("select", "bwd_rows", "bwd_items") else "hbm"
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
        if paths & _lib.PATH_WINDOW_FMA:
            src.update(select=["window_fma.cu", "window.cu"],
                       bwd_rows=["backward.cu", "window_fma.cu"], bwd_items=["window_fma.cu"])
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
        if self.index is None:  # not sampled
            return self
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
def oracle_rate():
    """Multiply-adds per second of the CPU oracle's scoring loops on this host (a short
    bucketing run), used only to size the slices below."""
    import oracle
    rng = np.random.Generator(np.random.PCG64(7))
    V = rng.standard_normal((4096, 256), dtype=np.float32)
    B = rng.standard_normal((256, 256), dtype=np.float32)
    oracle.bucketize(V[:256], B)
    t0 = time.perf_counter()
    oracle.bucketize(V, B)
    return V.shape[0] * B.shape[0] * V.shape[1] / (time.perf_counter() - t0)


def oracle_slice(w, seconds, rate):
    """A proportional slice of workload w for the CPU oracle: N, C and n_c divided by the
    same power of two f, so that chunks keep their sizes (N/n_c rows, C/n_c items) and
    rows keep their windows, their n_b projections and their k; each row's and item's
    work is then that of the whole workload (bar the clipped windows of the two end
    chunks), and the slice's rows/s stands for the whole workload's.  f is the smallest
    that brings the slice's multiply-adds (bucketing plus window scores) within `seconds`
    at `rate`, keeping n_c >= 8; f = 1 (the workload itself) when it fits."""
    from reduced_cross_entropy_b200 import synth

    def fmaf(N, C, n_c):
        ws = synth.Workload(w.name, N=N, d=w.d, C=C, dtype=w.dtype, n_b=w.n_b, n_c=n_c,
                            n_ec=w.n_ec, n_r=w.n_r, k=w.k)
        return (N + C) * w.n_b * w.d * w.n_r + pairs_per_round(ws) * w.d * w.n_r

    f = 1
    while (fmaf(w.N // f, w.C // f, w.n_c // f) > seconds * rate and w.n_c // (2 * f) >= 8
           and w.N % (2 * f) == 0 and w.C % (2 * f) == 0 and w.n_c % (2 * f) == 0):
        f *= 2
    if f == 1:
        return w, 1
    return w.scaled(w.N // f, w.C // f, n_c=w.n_c // f), f


def mean_window(w):
    """Window items per row, averaged over the rows (edge chunks see clipped windows)."""
    return pairs_per_round(w) / max(w.N, 1)


def oracle_step(ws, X, Y, t, B, all_negatives=False):
    """One whole step of the CPU oracle on workload ws (bucketing, stable sorts, the
    selection or Algorithm 1's window sums, loss, gradients); returns its seconds."""
    import oracle
    t0 = time.perf_counter()
    bx = [oracle.bucketize(X, B[r]) for r in range(ws.n_r)]
    by = [oracle.bucketize(Y, B[r]) for r in range(ws.n_r)]
    px = np.stack([oracle.stable_argsort(b) for b in bx])
    py = np.stack([oracle.stable_argsort(b) for b in by])
    if all_negatives:  # Algorithm 1 as printed: every window item a negative
        _, _, lse = oracle.window_loss(X, Y, t, px, py, ws.n_c, ws.n_ec)
        oracle.window_grad(X, Y, t, px, py, ws.n_c, ws.n_ec, lse, 1.0)
    else:
        sel, _, _ = oracle.select(X, Y, t, px, py, ws.n_c, ws.n_ec, ws.k)
        _, _, lse = oracle.rece_loss(X, Y, t, sel)
        oracle.rece_grad(X, Y, t, sel, lse, 1.0)
    return time.perf_counter() - t0


def oracle_sample_desc(w, ws, f):
    if f == 1:
        return f"the whole workload ({w.N} rows, {w.C} items): the oracle's full step, timed"
    return (f"a 1/{f} slice of the workload, its whole step timed: N={ws.N} rows, C={ws.C} "
            f"items, n_c={ws.n_c} (chunks of {w.N // w.n_c} rows and {w.C / w.n_c:g} items; "
            f"n_b, d, k, n_ec as in the workload; {mean_window(ws):.0f} window items per row "
            f"against the workload's {mean_window(w):.0f}); the slice's rows/s is reported "
            f"for the whole workload (extrapolated, linear in N and C)")


def oracle_projections(ws, seed, step):
    """The oracle's draw of a step's random vectors (the library's stream), in the
    workload's element type."""
    import oracle
    from reduced_cross_entropy_b200 import synth
    B = oracle.draw_projections(seed, step, ws.n_r, ws.n_b, ws.d)
    return synth.round_bf16(B) if ws.dtype == "bf16" else B


def cpu_baseline(w, seed, all_negatives=False, seconds=20.0):
    """rows/s of the CPU oracle on workload w (or its proportional slice), one step of
    about `seconds`."""
    import oracle
    from reduced_cross_entropy_b200 import synth
    ws, f = oracle_slice(w, seconds, oracle_rate())
    X, Y, t = synth.make_inputs(ws, seed=seed)
    sec = oracle_step(ws, X, Y, t, oracle_projections(ws, 0, 0), all_negatives)
    return {"value": ws.N / sec, "unit": "rows/s", "cores": oracle.num_threads(),
            "kind": "oracle", "method": "extrapolated" if f > 1 else "full",
            "sample": oracle_sample_desc(w, ws, f), "seconds": sec}


def run_reference(args):
    rank, _, _ = dist_env()
    if rank != 0:  # the oracle arm runs on rank 0 alone; other ranks exit without work
        return
    import oracle
    from reduced_cross_entropy_b200 import synth
    w = synth.WORKLOADS[args.workload]
    # every step is one whole oracle step on a slice sized so that all warm-up and timed
    # steps take about two minutes
    ws, f = oracle_slice(w, 120.0 / max(args.steps + args.warmup, 1), oracle_rate())
    X, Y, t = synth.make_inputs(ws, seed=0)
    alln = bool(getattr(args, "flags", 0) & 0x2)  # RECE_FLAG_ALL_NEGATIVES: Algorithm 1 as printed
    for s in range(args.warmup):
        oracle_step(ws, X, Y, t, oracle_projections(ws, 0, s), alln)
    secs = [oracle_step(ws, X, Y, t, oracle_projections(ws, 0, args.warmup + s), alln)
            for s in range(args.steps)]
    total = sum(secs)
    value = ws.N * args.steps / total  # each step is the slice's whole step: ws.N rows
    cores = oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * total / args.steps, "rows_per_step": ws.N,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(w)},
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": cores, "kind": "oracle",
                             "method": "extrapolated" if f > 1 else "full",
                             "sample": oracle_sample_desc(w, ws, f)},
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
class WorkloadRun:
    """One workload on one GPU: seeded inputs resident in HBM, a plan, its workspace and
    outputs, and the step (rece_bucketize_sort + rece_loss_fwd + rece_loss_bwd, and the
    ranks' dY exchange when there is one) timed with CUDA events on the launching stream."""

    def __init__(self, torch, w, seed, dev, flags, n_steps, exchange):
        from reduced_cross_entropy_b200 import _lib, ops, synth
        self.torch, self.w, self.dev, self.exchange = torch, w, dev, exchange
        self.L, self._lib = _lib.lib(), _lib
        self.X, self.Y, self.t = synth.make_inputs(w, seed=seed)
        self.tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype,
                             flags=flags)
        self.paths = self.plan.paths
        self.Xd = torch.from_numpy(self.X).to(dev).to(self.tdt)
        self.Yd = torch.from_numpy(self.Y).to(dev).to(self.tdt)
        self.td = torch.from_numpy(self.t).to(dev)
        # B is drawn afresh on the device in every step (the method's randn inside the
        # loss, rece_draw_projections), keyed by (seed 0, step) on every rank so that the
        # replicas bucket alike
        self.Bd = torch.empty((w.n_r, w.n_b, w.d), dtype=self.tdt, device=dev)
        self.n_steps = n_steps
        self.ws = self.plan.workspace(dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.loss = torch.empty(1, **f32)
        self.sel = torch.empty(w.N, w.k, dtype=torch.int32, device=dev)
        self.lse = torch.empty(w.N, **f32)
        self.logits = torch.empty(w.N, w.k + 1, **f32)
        self.dloss = torch.ones(1, **f32)
        self.dX = torch.empty(w.N, w.d, **f32)
        self.dY = torch.empty(w.C, w.d, **f32)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.sp = ctypes.c_void_p(self.stream.cuda_stream)
        self.nbytes = ctypes.c_size_t(self.ws.numel())

    def step(self, s, Xc=None, Yc=None, tc=None):
        vp = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
        L, h, sp, ck = self.L, self.plan._h, self.sp, self._lib.check
        Xc = self.Xd if Xc is None else Xc
        Yc = self.Yd if Yc is None else Yc
        tc = self.td if tc is None else tc
        ck(L.rece_draw_projections(h, 0, s, vp(self.Bd), sp), "draw_projections")
        ck(L.rece_bucketize_sort(h, vp(self.Bd), vp(Xc), vp(Yc), vp(self.ws), self.nbytes, sp),
           "bucketize_sort")
        ck(L.rece_loss_fwd(h, vp(Xc), vp(Yc), vp(tc), vp(self.ws), self.nbytes, vp(self.loss),
                           None, vp(self.sel), vp(self.lse), vp(self.logits), sp), "loss_fwd")
        ck(L.rece_loss_bwd(h, vp(Xc), vp(Yc), vp(tc), vp(self.sel), vp(self.lse),
                           vp(self.logits), vp(self.dloss), vp(self.ws), self.nbytes,
                           vp(self.dX), vp(self.dY), sp), "loss_bwd")
        if self.exchange:
            allreduce_dy(self.dY)

    def warm(self, warmup):
        for s in range(warmup):
            self.flush.zero_()
            self.step(s)
        self.torch.cuda.synchronize(self.dev)
        # status area: flags (a bad target or a timed-out wait fails the run; the
        # tensor-core selection may flag rows it cannot certify exact) and row counts
        words = self.ws[:32].view(self.torch.int32).cpu().tolist()
        assert words[0] & ~self._lib.DEVICE_INEXACT == 0, f"device status {words[0]:#x}"
        self.status_words = {"inexact_rows_per_step": int(words[1]),
                             "overflowed_rows_per_step": int(words[2]),
                             "merge_spilled_rows_per_step": int(words[3])}
        if self.paths & self._lib.PATH_SAMPLED_SELECT:
            # work items (128 rows of a round) the sampled selection could not certify
            # and handed to the exact kernel
            self.status_words["select_redo_items_per_step"] = int(words[4])

    def timed(self, first, steps, barrier=lambda: None, clock_index=None):
        """`steps` steps from B number `first`, L2 flushed before each; per-step and
        per-stage CUDA events (the library records the stage events on the same stream).
        Returns (per-step ms, mean ms per stage, kernel launches, clock summary)."""
        torch, _lib, stream = self.torch, self._lib, self.stream
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        n_st = len(_lib.STAGES)
        sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n_st)]
               for _ in range(steps)]
        for row in sev:  # torch creates the CUDA event at its first record
            for e in row:
                e.record(stream)
        sev_h = [(ctypes.c_void_p * (2 * n_st))(*[ctypes.c_void_p(e.cuda_event) for e in row])
                 for row in sev]
        launches0 = self.L.rece_kernel_launch_count()
        barrier()
        torch.cuda.synchronize(self.dev)
        with ClockSampler(clock_index) as clk:
            for s in range(steps):
                self.flush.zero_()
                _lib.check(self.L.rece_plan_set_stage_events(self.plan._h, sev_h[s]),
                           "stage events")
                ev[s][0].record(stream)
                self.step(first + s)
                ev[s][1].record(stream)
            torch.cuda.synchronize(self.dev)
        barrier()
        launches = self.L.rece_kernel_launch_count() - launches0
        self.L.rece_plan_set_stage_events(self.plan._h, None)
        step_ms = [a.elapsed_time(b) for a, b in ev]
        stage_ms = {name: statistics.mean(sev[s][2 * i].elapsed_time(sev[s][2 * i + 1])
                                          for s in range(steps))
                    for i, name in enumerate(_lib.STAGES)}
        return step_ms, stage_ms, launches, (clk.summary() if clock_index is not None else None)

    def rooflines(self, stage_ms):
        """(roofline of the dominant stage, every stage's fraction of its roofline)."""
        peaks = load_peaks()
        work = stage_work(self.w, self.paths)

        def one(name):
            bound = stage_bound(name, self.paths)
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
                    "traffic": recorded_traffic(name, self.w.name, self.paths),
                    "algorithmic_bytes": bytes_, "algorithmic_flops": flops}

        dom = max(stage_ms, key=stage_ms.get)
        return one(dom), {name: round(one(name)["frac"], 4) for name in stage_ms}

    def path_roofline(self, ms_per_step):
        """The whole step against the sum of every stage's roofline time."""
        peaks = load_peaks()
        t = 0.0
        for name, (flops, bytes_) in stage_work(self.w, self.paths).items():
            t += max(flops / (peaks["bf16_tflops"] * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9))
        return {"roofline_ms": 1000 * t, "measured_ms": ms_per_step,
                "frac": 1000 * t / ms_per_step}

    def describe(self):
        _lib, w, paths = self._lib, self.w, self.paths
        return {"workload": workload_desc(w), **self.status_words,
                "l2": "flushed between timed steps (256 MiB write)",
                "scores": ("tcgen05" + (", stored" if paths & _lib.PATH_STORED_SCORES
                                          else ", threshold from a 1/8 sample, one pass"
                                          if paths & _lib.PATH_SAMPLED_SELECT
                                          else ", exact threshold, three passes")
                           if paths & _lib.PATH_TENSOR_CORES else "fmaf CUDA cores"),
                "dX": ("tcgen05 band products" +
                       (", rounds in one launch, parts summed in order"
                        if paths & _lib.PATH_DX_PARTS else "")
                       if paths & _lib.PATH_DX_TENSORS else "gathered rows"),
                "dY": ("tcgen05 band products" if paths & _lib.PATH_DY_TENSORS
                       else "pairs sorted by item, gathered rows"),
                "negatives": ("every window item (Algorithm 1 as printed), window "
                              "sums and gradients on tcgen05"
                              if paths & _lib.PATH_ALL_NEGATIVES else f"top-{w.k} per row")}

    def e2e(self, warmup, steps, barrier=lambda: None):
        """End to end through the same C-ABI calls: every step's inputs copied in from
        pinned host memory and its loss copied out.  Step s+1's copies (a copy stream,
        two device input sets) overlap step s's compute, as a training input pipeline
        does; the L2 flush stays in the timeline; one pair of events spans all timed
        steps.  Returns (total ms of the timed steps, h2d bytes per step, d2h bytes)."""
        torch, dev, stream = self.torch, self.dev, self.stream
        tdt = self.tdt
        Xh = torch.from_numpy(self.X).to(tdt).pin_memory()
        Yh = torch.from_numpy(self.Y).to(tdt).pin_memory()
        th = torch.from_numpy(self.t).pin_memory()
        loss_h = torch.empty(self.n_steps, dtype=torch.float32).pin_memory()
        h2d = Xh.numel() * Xh.element_size() + Yh.numel() * Yh.element_size() + th.numel() * 4
        sets = [(self.Xd, self.Yd, self.td),
                (torch.empty_like(self.Xd), torch.empty_like(self.Yd),
                 torch.empty_like(self.td))]
        cstream = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        consumed = [torch.cuda.Event() for _ in range(2)]

        def issue_copy(s, j):
            k = s % 2
            with torch.cuda.stream(cstream):
                if j >= 2:  # the set's previous step has finished with it
                    cstream.wait_event(consumed[k])
                for dst, src in zip(sets[k], (Xh, Yh, th)):
                    dst.copy_(src, non_blocking=True)
                copied[k].record(cstream)

        def run(first, count):
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
                self.flush.zero_()
                Xc, Yc, tc = sets[k]
                self.step(s, Xc, Yc, tc)
                consumed[k].record(stream)
                loss_h[s].copy_(self.loss[0], non_blocking=True)
            t1.record(stream)
            t1.synchronize()
            return t0.elapsed_time(t1)

        run(0, warmup)
        barrier()
        ms = run(warmup, steps)
        assert np.all(np.isfinite(loss_h.numpy())), "non-finite loss"
        del sets
        return ms, int(h2d), 4


def extra_workload(torch, name, args, dev):
    """Another workload measured in the same process (one GPU): ms per step, rows/s, the
    dominant stage's roofline, every stage's fraction and peak HBM against full CE."""
    from reduced_cross_entropy_b200 import ops, synth
    w = synth.WORKLOADS[name]
    run = WorkloadRun(torch, w, 0, dev, args.flags, args.warmup + args.steps, False)
    run.warm(args.warmup)
    step_ms, stage_ms, launches, _ = run.timed(args.warmup, args.steps)
    ms = sum(step_ms) / args.steps
    roof, fracs = run.rooflines(stage_ms)
    out = {"config": run.describe(), "ms_per_step": ms, "value": w.N / (ms / 1000.0),
           "unit": "rows/s", "steps": args.steps, "warmup": args.warmup,
           "roofline": roof, "path_roofline": run.path_roofline(ms), "stages_ms": stage_ms,
           "stages_roofline_frac": fracs, "gpu_launches": int(launches)}
    if not args.no_memory:
        out["peak_hbm"] = measure_memory(torch, ops, run.plan, w, run.Xd, run.Yd, run.td,
                                         run.Bd, dev)
    del run
    torch.cuda.empty_cache()
    return out


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
    w = synth.WORKLOADS[args.workload]
    if args.slice > 1:
        f = args.slice
        if w.N % f or w.C % f or w.n_c % f:
            raise SystemExit(f"--slice {f} must divide N, C and n_c of {w.name}")
        w = w.scaled(w.N // f, w.C // f, n_c=w.n_c // f)
    run = WorkloadRun(torch, w, rank, dev, args.flags, args.warmup + args.steps, exchange)
    run.warm(args.warmup)
    step_ms, stage_ms, launches, clocks = run.timed(args.warmup, args.steps, barrier,
                                                    clock_index=local_rank)
    total_ms = max_over_ranks(sum(step_ms), dev)
    value = job_throughput(world, w.N, args.steps, total_ms)
    roofline, stage_fracs = run.rooflines(stage_ms)
    e2e_ms, h2d, d2h = run.e2e(args.warmup, args.steps, barrier)
    e2e_total = max_over_ranks(e2e_ms, dev)
    e2e = {"value": job_throughput(world, w.N, args.steps, e2e_total), "unit": "rows/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    paths = run.paths
    config = run.describe()
    config.update({"parallelism": f"dp{world}",
                   "exchange": ("all-reduce of dY [C x d] fp32 every step (NCCL)"
                                if exchange else "none")})
    line = {"metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": config, "roofline": roofline,
            "path_roofline": run.path_roofline(total_ms / args.steps),
            "stages_ms": stage_ms, "stages_roofline_frac": stage_fracs,
            "e2e": e2e, "gpu_launches": int(launches), "clocks": clocks}

    if rank == 0 and world == 1 and not args.no_memory:
        line["peak_hbm"] = measure_memory(torch, ops, run.plan, w, run.Xd, run.Yd, run.td,
                                          run.Bd, dev)
    if rank == 0 and world == 1 and not args.no_baselines:
        line["baselines"] = measure_baselines(torch, ops, w, run.Xd, run.Yd, run.td, run.flush,
                                              dev, load_peaks())
    del run
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and args.also:
        line["workloads"] = {name: extra_workload(torch, name, args, dev)
                             for name in args.also.split(",") if name and name != w.name}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, 0, bool(paths & _lib.PATH_ALL_NEGATIVES))
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

    fused_ms = []

    def fused():
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        _, _, l, ws = ops.full_ce_fwd(Xd, Yd, td)
        ops.full_ce_bwd(Xd, Yd, td, l, torch.ones(1, device=dev), ws)
        b.record()
        b.synchronize()
        fused_ms.append(a.elapsed_time(b))

    out["rece_bytes"] = peak(rece)
    # the fused exact op's memory is its outputs (lse, row losses, dX, dY in fp32) and its
    # workspace, whatever the run time; it is run where its 6 N C d flops take seconds
    ws_bytes = ops.full_ce_workspace_bytes(w.N, w.C, w.d, w.dtype)
    out["full_ce_fused_bytes_computed"] = 4 * (2 * w.N + w.N * w.d + w.C * w.d + 1) + ws_bytes
    # the op runs on tcgen05 for bf16 with d a multiple of 64 up to 256, else on the CUDA
    # cores (measured: about 112 s for one fwd+bwd at N = 16,384, C = 128,000, d = 4096):
    # run it (and time one fwd+bwd, after one untimed) where that takes seconds
    tc = w.dtype == "bf16" and w.d % 64 == 0 and w.d <= 256
    if 6.0 * w.N * w.C * w.d <= (2e15 if tc else 3e13):
        fused()
        out["full_ce_fused_bytes"] = peak(fused)
        out["full_ce_fused_ms_fwd_bwd"] = fused_ms[-1]
        out["full_ce_fused_kernels"] = "tcgen05" if tc else "CUDA cores"
    else:
        out["full_ce_fused_bytes"] = None
        out["full_ce_fused_note"] = (f"not run: {6.0 * w.N * w.C * w.d:.1e} flops; its allocations "
                                     f"are full_ce_fused_bytes_computed")
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
    fused_ref = out["full_ce_fused_bytes"] or out["full_ce_fused_bytes_computed"]
    out["ratio_vs_fused"] = fused_ref / max(out["rece_bytes"], 1)
    # the pages' memory model of Algorithm 1 (every chunk's logits stored) at this
    # workload's alpha_bc = n_b / n_c, and the bucket count it calls optimal
    a = w.n_b / w.n_c
    nb, nc = ops.optimal_buckets(w.N, w.C, w.n_ec, a)
    el = ops.memory_model_elements(w.N, w.C, w.n_ec, w.n_r, a)
    out["pages_memory_model"] = {"alpha_bc": a, "n_b_star": nb, "n_c_star": nc,
                                 "logit_elements": el, "bytes_fp32": 4 * el,
                                 "rece_bytes_over_model": out["rece_bytes"] / (4 * el)}
    # the plan the library makes when asked for the pages' optimum (n_b = n_c = 0:
    # n_b* at alpha_bc = 1) and its workspace, against the model at alpha_bc = 1
    auto = ops.Plan(w.N, w.C, w.d, 0, 0, w.n_ec, w.n_r, w.k, mode=w.dtype,
                    flags=plan.cfg.flags)
    el1 = ops.memory_model_elements(w.N, w.C, w.n_ec, w.n_r, 1.0)
    out["pages_memory_model"]["auto_plan"] = {
        "n_b": auto.n_b, "n_c": auto.n_c, "workspace_bytes": auto.workspace_bytes,
        "model_bytes_fp32": 4 * el1, "workspace_over_model": auto.workspace_bytes / (4 * el1)}
    out["note"] = "bytes above the resident inputs; torch.cuda.max_memory_allocated"
    return out


if __name__ == "__main__":
    main()
