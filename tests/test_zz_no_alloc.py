"""The allocation-free bucket sort, rece_bucket_sort_static, called through the C ABI.

Some callers cannot give the library device memory: code inside another application's
fixed device-memory arena, or a loop that cannot take an allocation's latency.  This
entry point keeps the sort's scratch in a fixed array inside the library.  Its output
must equal the workspace-based sort of rece_bucketize_sort, call after call, although
every call reuses the same scratch.  (This file is collected last on purpose.)
"""
import ctypes

import numpy as np
import pytest
import torch

from reduced_cross_entropy_b200 import _lib, ops, synth
from tests.gpu_common import to_dev

pytestmark = pytest.mark.gpu


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def test_static_sort_matches_workspace_sort():
    w = synth.WORKLOADS["sasrec"].scaled(3200, 12500, n_c=8)
    X, Y, t = synth.make_inputs(w, seed=4)
    B = synth.projections(4, 0, w.n_r, w.n_b, w.d, w.dtype)
    plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype)
    ws = plan.workspace()
    ops.bucketize_sort(plan, to_dev(B, w.dtype), to_dev(X, w.dtype), to_dev(Y, w.dtype), ws)
    bx, by = plan.bucket_ids(ws)
    px, py = plan.permutations(ws)
    starts_y = plan.bucket_starts_y(ws)
    torch.cuda.synchronize()

    L = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    stride = plan.layout.bucket_start_stride
    # several calls in a row, large then small then large again: the shared scratch
    # keeps the previous call's contents and must not leak into the next result
    calls = [(by[0], py[0], starts_y[0]), (bx[0], px[0], None), (by[1], py[1], starts_y[1]),
             (bx[1], px[1], None)]
    for keys, want, want_starts in calls:
        keys = keys.contiguous()
        M = keys.numel()
        order = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        starts = torch.full((stride,), -7, dtype=torch.int32, device="cuda")
        s = L.rece_bucket_sort_static(_vp(keys), M, w.n_b, _vp(order), _vp(starts), stream)
        assert s == 0, L.rece_last_error_string()
        torch.cuda.synchronize()
        assert torch.equal(order, want)
        if want_starts is not None:
            assert torch.equal(starts, want_starts)
        np.testing.assert_array_equal(order.cpu().numpy(),
                                      np.argsort(keys.cpu().numpy(), kind="stable"))


def test_static_sort_rejects_sizes_beyond_its_scratch():
    L = _lib.lib()
    keys = torch.zeros(16, dtype=torch.int32, device="cuda")
    order = torch.empty(16, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # rejected on the host before anything is launched (the pointers are never read)
    s = L.rece_bucket_sort_static(_vp(keys), 1 << 28, 4096, _vp(order), None, stream)
    assert s == 2
    assert b"4 MiB" in L.rece_last_error_string()
    assert L.rece_bucket_sort_static(_vp(keys), 16, 0, _vp(order), None, stream) == 1
    # a size that fits still works after the rejection
    s = L.rece_bucket_sort_static(_vp(keys), 16, 4096, _vp(order), None, stream)
    assert s == 0
    torch.cuda.synchronize()
    assert torch.equal(order, torch.arange(16, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("M,n_b", [(5000, 300), (2048 * 3 + 17, 4096), (1, 1), (777, 2)])
def test_static_sort_out_of_range_keys_sort_by_their_low_bits(M, n_b):
    # hand-made keys: in range, at and above n_b, and negative; M off the 2048-element tile
    rng = np.random.Generator(np.random.PCG64(M + n_b))
    keys = rng.integers(-3 * n_b - 5, 3 * n_b + 5, size=M).astype(np.int32)
    keys[: min(M, 4)] = np.array([-1, n_b, -2147483648, 2147483647][: min(M, 4)], np.int32)
    bits = max(int(np.ceil(np.log2(n_b))), 0) if n_b > 1 else 0
    digit = (keys.astype(np.int64) & ((1 << bits) - 1)).astype(np.int64)
    want = np.argsort(digit, kind="stable").astype(np.int32)
    stride = (1 << bits) + 1
    want_starts = np.searchsorted(digit[want], np.arange(stride), side="left").astype(np.int32)

    L = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    kd = torch.from_numpy(keys).cuda()
    for _ in range(2):  # twice in a row: the shared scratch keeps the first call's contents
        order = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        starts = torch.full((stride,), -7, dtype=torch.int32, device="cuda")
        s = L.rece_bucket_sort_static(_vp(kd), M, n_b, _vp(order), _vp(starts), stream)
        assert s == 0, L.rece_last_error_string()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(order.cpu().numpy(), want)
        np.testing.assert_array_equal(starts.cpu().numpy(), want_starts)
