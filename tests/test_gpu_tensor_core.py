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


@pytest.mark.parametrize("d,n_b", [(64, 16), (64, 256), (128, 300), (192, 1024), (64, 1),
                                   (256, 2048), (256, 2100)])
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


# ---------------------------------------------------------------- whole path, tcgen05
TC_CASES = {
    "tiny_bf16_rounds2": synth.WORKLOADS["tiny"].scaled(256, 4096, dtype="bf16", n_r=2, k=40),
    "sasrec_scaled": synth.WORKLOADS["sasrec"].scaled(3200, 12500, n_c=8),
    "sasrec_scaled_2": synth.WORKLOADS["sasrec"].scaled(6400, 25000, n_c=16),
    "large_norms_scaled": synth.WORKLOADS["large"].scaled(2000, 20000, n_c=10, n_b=128, k=128),
    "lm_scaled": synth.WORKLOADS["lm"].scaled(512, 4000, n_c=4, n_b=64, k=128, d=256),
    "very_large_scaled": synth.WORKLOADS["very_large"].scaled(4096, 40000, n_c=64, n_b=256,
                                                              k=256),
    # d >= 1024: window scores computed once and stored, then selected row by row
    "lm_scaled_d1024": synth.WORKLOADS["lm"].scaled(512, 4000, n_c=4, n_b=64, k=128, d=1024),
}


def recall(sel_gpu, sel_orc):
    hit = tot = 0
    for a, b in zip(sel_gpu, sel_orc):
        sb = set(b[b >= 0].tolist())
        hit += len(sb & set(a[a >= 0].tolist()))
        tot += len(sb)
    return hit / max(tot, 1)


@pytest.mark.parametrize("name", sorted(TC_CASES))
def test_tc_path_recall_and_loss(name):
    w = TC_CASES[name]
    X, Y, t = synth.make_inputs(w, seed=3)
    B = synth.projections(3, 0, w.n_r, w.n_b, w.d, "bf16")
    g = run_gpu(w, X, Y, t, B, flags=0, dloss=1.0)
    o = run_oracle(w, X, Y, t, B, dloss=1.0)
    rc = recall(g["selected"], o["selected"])
    assert rc >= 0.99, rc
    assert abs(g["loss"] - o["loss"]) <= 1e-2 * abs(o["loss"])
    assert g["status"] & ~0x4 == 0
    # every row's kept negatives are distinct, never the positive, and inside its windows
    for i in range(0, w.N, max(1, w.N // 64)):
        s = g["selected"][i]
        s = s[s >= 0]
        assert len(set(s.tolist())) == len(s) and t[i] not in set(s.tolist())
    # gradients of the selection the GPU made, against the oracle's fp64 formula
    _, _, lse = oracle.rece_loss(X, Y, t, g["selected"])
    oX, oY = oracle.rece_grad(X, Y, t, g["selected"], lse, 1.0)
    assert max_rel(g["dX"], oX) <= 1e-3
    assert max_rel(g["dY"], oY) <= 1e-3


@pytest.mark.parametrize("d,n_c,n_ec,n_r,k", [(64, 8, 1, 2, 64), (64, 16, 0, 1, 200),
                                              (128, 6, 2, 3, 100), (256, 8, 1, 2, 96),
                                              (1024, 8, 1, 2, 96), (64, 8, 1, 2, 600),
                                              (256, 8, 1, 1, 600)])
def test_tc_path_exact_on_integer_inputs(d, n_c, n_ec, n_r, k):
    """Integer-valued inputs: every score is exact on the tensor cores and ties are
    everywhere, so the kept sets (ties to the lower item id) must be the oracle's.  At
    d >= 256 dX also comes from the tensor cores (band products of the coefficients); at
    d = 1024 the window scores are stored once and selected row by row.  At k >= 512 the
    merge spreads each row over four warps."""
    w = synth.Workload("int", N=1000, C=5003, d=d, dtype="bf16", n_b=16, n_c=n_c, n_ec=n_ec,
                       n_r=n_r, k=k)
    X, Y, t = synth.integer_inputs(w.N, w.C, d, lo=-2, hi=2, seed=d + k, scale=0.125)
    B = synth.integer_inputs(n_r * w.n_b, 1, d, lo=-2, hi=2, seed=k, scale=1.0)[0]
    B = B.reshape(n_r, w.n_b, d)
    g = run_gpu(w, X, Y, t, B, flags=0, dloss=0.5)
    o = run_oracle(w, X, Y, t, B, dloss=0.5)
    assert g["status"] == 0
    print("rows spilled to the merge's global-memory path:", int(g["words"][3]))
    np.testing.assert_array_equal(np.sort(g["selected"], axis=1), np.sort(o["selected"], axis=1))
    assert abs(g["loss"] - o["loss"]) <= 1e-4 * abs(o["loss"])
    assert max_rel(g["row_loss"], o["row_loss"]) <= 1e-4
    assert max_rel(g["dX"], o["dX"]) <= 1e-4 and max_rel(g["dY"], o["dY"]) <= 1e-4
    # the logits output is the positive's and each kept item's exact score
    lg, sel = g["logits"], g["selected"]
    np.testing.assert_array_equal(lg[:, 0], np.einsum("nd,nd->n", X, Y[t]))
    for i in range(0, w.N, 37):
        s = sel[i][sel[i] >= 0]
        np.testing.assert_array_equal(lg[i, 1:1 + len(s)], Y[s] @ X[i])
        assert np.all(lg[i, 1 + len(s):] == -np.inf)


def test_backward_past_the_in_cache_pair_size():
    """N (k+1) > 8.4M pairs: the pair sort carries each pair's coefficient instead of the
    item pass gathering it.  Gradients against the oracle's, for the GPU's selection."""
    w = synth.WORKLOADS["sasrec"].scaled(33_000, 100_000)
    assert w.N * (w.k + 1) * 4 > (32 << 20)
    X, Y, t = synth.make_inputs(w, seed=6)
    B = synth.projections(6, 0, w.n_r, w.n_b, w.d, "bf16")
    g = run_gpu(w, X, Y, t, B, flags=0, dloss=0.5)
    assert g["status"] & ~0x4 == 0
    _, _, lse = oracle.rece_loss(X, Y, t, g["selected"])
    oX, oY = oracle.rece_grad(X, Y, t, g["selected"], lse, 0.5)
    assert max_rel(g["dX"], oX) <= 1e-3
    assert max_rel(g["dY"], oY) <= 1e-3


@pytest.mark.parametrize("d", [64, 256])
def test_merge_spill_path_on_tied_scores(d):
    """Every score equal: each row's whole window is emitted (one histogram bin, about 500
    positions), more candidates than the merge's shared-memory buffers, so the rows go
    through the spill path (global-memory buffers).  Ties go to the lower item id: the oracle's sets."""
    w = synth.Workload("tied", N=300, C=1000, d=d, dtype="bf16", n_b=8, n_c=6, n_ec=1,
                       n_r=1, k=100)
    X = np.full((w.N, d), 0.125, np.float32)
    Y = np.full((w.C, d), 0.25, np.float32)
    t = np.random.default_rng(5).integers(0, w.C, w.N).astype(np.int32)
    B = synth.projections(5, 0, w.n_r, w.n_b, d, "bf16")
    g = run_gpu(w, X, Y, t, B, flags=0, dloss=1.0)
    o = run_oracle(w, X, Y, t, B, dloss=1.0)
    assert g["status"] == 0
    assert g["words"][3] > 0  # rows that took the spill path
    np.testing.assert_array_equal(np.sort(g["selected"], axis=1), np.sort(o["selected"], axis=1))
    assert abs(g["loss"] - o["loss"]) <= 1e-4 * abs(o["loss"])
    # with every y equal, dX_i = y * sum_j g_ij vanishes (the softmax sums to 1): measure
    # it against the size of its terms, dloss / N * |y|
    term = 1.0 / w.N * float(np.abs(Y).max())
    assert np.abs(g["dX"] - o["dX"]).max() <= 1e-4 * term
    assert max_rel(g["dY"], o["dY"]) <= 1e-4


def test_merge_four_warp_rows_spill_on_tied_scores():
    """k >= 512: each row is merged by four warps, each holding one selection sub-list.
    Every score tied (x = e_0, y_0 = 1/4, the other coordinates of y random, so the
    catalogue's buckets still differ from round to round): each round emits its whole
    window, about 1930 positions, and two rounds' entries overfill the warps' regions, so
    rows go through the spill path.  Ties go to the lower item id: the oracle's sets."""
    w = synth.Workload("tied4", N=300, C=9000, d=64, dtype="bf16", n_b=8, n_c=14, n_ec=1,
                       n_r=2, k=512)
    X = np.zeros((w.N, w.d), np.float32)
    X[:, 0] = 1.0
    rng = np.random.default_rng(12)
    Y = rng.integers(-2, 3, (w.C, w.d)).astype(np.float32) * 0.125
    Y[:, 0] = 0.25
    t = rng.integers(0, w.C, w.N).astype(np.int32)
    # integer projections: every projection exact on both sides, ties to the lower bucket
    B = synth.integer_inputs(w.n_r * w.n_b, 1, w.d, lo=-2, hi=2, seed=12, scale=1.0)[0]
    B = B.reshape(w.n_r, w.n_b, w.d)
    g = run_gpu(w, X, Y, t, B, flags=0, dloss=1.0)
    o = run_oracle(w, X, Y, t, B, dloss=1.0)
    assert g["status"] == 0
    assert g["words"][3] > 0  # rows that took the spill path
    np.testing.assert_array_equal(np.sort(g["selected"], axis=1), np.sort(o["selected"], axis=1))
    assert abs(g["loss"] - o["loss"]) <= 1e-4 * abs(o["loss"])
    assert max_rel(g["dX"], o["dX"]) <= 1e-4 and max_rel(g["dY"], o["dY"]) <= 1e-4


def test_sampled_selection_hands_misled_rows_to_the_exact_kernel():
    """d >= 256: each row's threshold comes from a sample of its window (the first 16
    positions of every 128-position tile).  With one bucket the sorted order is the item
    order, so making exactly the sampled items score high misleads the sample: fewer than
    k + 1 scores pass its threshold, the rows cannot be certified and go to the exact
    three-pass kernel.  The kept sets must still be the oracle's (ties to the lower id)."""
    from reduced_cross_entropy_b200 import _lib
    w = synth.Workload("misled", N=256, C=4096, d=256, dtype="bf16", n_b=1, n_c=2, n_ec=0,
                       n_r=1, k=400)
    X = np.full((w.N, w.d), 0.125, np.float32)
    j = np.arange(w.C)
    sampled = (j % 128) < 16
    Y = np.where(sampled[:, None], 0.25 * (1 + j[:, None] % 3), 0.125 * (j[:, None] % 5 - 2))
    Y = np.ascontiguousarray(np.broadcast_to(Y, (w.C, w.d)), dtype=np.float32)
    t = np.random.default_rng(9).integers(0, w.C, w.N).astype(np.int32)
    B = np.ones((1, 1, w.d), np.float32)
    g = run_gpu(w, X, Y, t, B, flags=0, dloss=1.0)
    assert g["plan"].paths & _lib.PATH_SAMPLED_SELECT
    assert g["status"] & ~0x4 == 0 and g["words"][1] == 0   # certified exact
    assert g["words"][4] > 0                                 # items redone exactly
    o = run_oracle(w, X, Y, t, B, dloss=1.0)
    np.testing.assert_array_equal(np.sort(g["selected"], axis=1), np.sort(o["selected"], axis=1))
    assert abs(g["loss"] - o["loss"]) <= 1e-4 * abs(o["loss"])
    assert max_rel(g["dX"], o["dX"]) <= 1e-4 and max_rel(g["dY"], o["dY"]) <= 1e-4
