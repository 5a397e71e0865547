"""Host logic of bench.py's multi-GPU run, on CPU ranks over gloo (world size 2).

Data-parallel replicas: every rank runs the whole loss on its own batch against the
shared catalogue (weak scaling), the ranks sum their dY once per step, and the job's time
is the slowest rank's.  These tests run that exchange, the timing reduction, the
throughput formula and the reference arm's rank rule as two gloo processes, no GPU
involved.
"""
import contextlib
import importlib.util
import io
import os
import socket
import types

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        assert bench.dist_env() == (rank, rank, world)
        # each rank's own total time; the job is as slow as its slowest rank
        mine = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(mine)
        # the data-parallel exchange: every rank ends with the sum of the ranks' dY
        import torch
        dY = torch.full((5, 3), float(rank + 1))
        bench.allreduce_dy(dY)
        assert torch.equal(dY, torch.full((5, 3), float(world * (world + 1) // 2)))
        rows = bench.job_throughput(world, 25_600, 4, slowest)
        # the reference (oracle) arm: rank 0 alone works and prints
        buf = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(types.SimpleNamespace(workload="tiny", warmup=0, steps=1,
                                                          gpus=world))
        out.put((rank, slowest, rows, buf.getvalue()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    got = sorted(out.get(timeout=60) for _ in range(world))
    for rank, slowest, rows, printed in got:
        assert slowest == 15.0                       # max over ranks, on every rank
        assert rows == pytest.approx(2 * 25_600 * 4 / 0.015)
        if rank != 0:
            assert printed == ""                     # non-zero ranks exit without work


def test_single_process_needs_no_group():
    bench = _bench()
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 100, 2, 1000.0) == pytest.approx(200.0)
