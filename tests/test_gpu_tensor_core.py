"""Parity of the tcgen05 (tensor-core) kernels of the bf16 mode with the CPU oracle.

The tensor cores accumulate in fp32 in their own order, so results can differ from the
oracle's fixed fmaf chain only where two scores are within rounding of each other:
* on integer-valued inputs every product and partial sum is exact, so bucket ids, sort
  orders and selections must match the oracle bit for bit;
* on random inputs every disagreement must be a near-tie, selected-set recall must be
  >= 0.99 and the loss within 1e-2 relative (the bar of the bf16 mode).
"""
import numpy as np
import pytest
import torch

import oracle
from reduced_cross_entropy_b200 import ops, synth
from tests.gpu_common import max_rel, run_gpu, run_oracle, to_dev

pytestmark = pytest.mark.gpu


def bucket_ids_gpu(w, X, Y, B):
    plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode="bf16")
    ws = plan.workspace()
    ops.bucketize_sort(plan, to_dev(B, "bf16"), to_dev(X, "bf16"), to_dev(Y, "bf16"), ws)
    bx, by = (a.cpu().numpy() for a in plan.bucket_ids(ws))
    px, py = (a.cpu().numpy() for a in plan.permutations(ws))
    assert ops.device_status(ws) == 0
    return bx, by, px, py


@pytest.mark.parametrize("d,n_b", [(64, 16), (64, 256), (128, 300), (192, 1024), (64, 1)])
def test_bucketize_tc_exact_on_integer_inputs(d, n_b):
    w = synth.Workload("int", N=1000, C=3001, d=d, dtype="bf16", n_b=n_b, n_c=4, n_ec=1,
                       n_r=2, k=8)
    X, Y, _ = synth.integer_inputs(w.N, w.C, d, lo=-2, hi=2, seed=d + n_b, scale=1.0)
    B = synth.integer_inputs(w.n_r * n_b, 1, d, lo=-2, hi=2, seed=7, scale=1.0)[0]
    B = B.reshape(w.n_r, n_b, d)
    bx, by, px, py = bucket_ids_gpu(w, X, Y, B)
    for r in range(w.n_r):
        np.testing.assert_array_equal(bx[r], oracle.bucketize(X, B[r]))
        np.testing.assert_array_equal(by[r], oracle.bucketize(Y, B[r]))
        np.testing.assert_array_equal(px[r], np.argsort(bx[r], kind="stable"))
        np.testing.assert_array_equal(py[r], np.argsort(by[r], kind="stable"))


def test_bucketize_tc_random_inputs_near_ties_only():
    w = synth.WORKLOADS["sasrec"].scaled(3200, 12500, n_c=8)
    X, Y, _ = synth.make_inputs(w, seed=1)
    B = synth.projections(1, 0, w.n_r, w.n_b, w.d, "bf16")
    bx, by, _, _ = bucket_ids_gpu(w, X, Y, B)
    for r in range(w.n_r):
        for V, got in ((X, bx[r]), (Y, by[r])):
            want = oracle.bucketize(V, B[r])
            diff = np.nonzero(got != want)[0]
            assert len(diff) <= 1e-3 * len(V)
            P = V[diff].astype(np.float64) @ B[r].astype(np.float64).T
            for row, i in enumerate(diff):
                a, b = P[row, got[i]], P[row, want[i]]
                assert abs(a - b) <= 1e-5 * np.abs(P[row]).max()
