"""Parity of the all-negatives mode -- Algorithm 1 of the RECE paper as printed (section 3):
every item of a row's chunk windows is a negative, a pair computed in cnt of the rounds
enters each round's sum as exp(l - ln cnt) -- on the tcgen05 kernels, through the C ABI,
against the oracle.

The oracle runs on the GPU's own bucket orders (checked to be stable sorts of the GPU's
bucket ids): tensor-core bucketing may settle a near-tie the other way, and the windows
follow the orders.  Values: lse and row losses within 1e-4, gradients within 1e-3 (the
tensor cores accumulate in fp32, P reaches them as hi + lo bf16)."""
import numpy as np
import pytest
import torch

import oracle
from reduced_cross_entropy_b200 import _lib, ops, synth
from tests.gpu_common import max_rel, to_dev

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = {
    "d64_rounds2": W("w1", N=700, C=3000, d=64, dtype="bf16", n_b=16, n_c=7, n_ec=1, n_r=2, k=8),
    "d128_one_round_no_neighbours": W("w2", N=517, C=2049, d=128, dtype="bf16", n_b=8, n_c=5,
                                      n_ec=0, n_r=1, k=8),
    "d256_rounds3_whole_catalogue": W("w3", N=300, C=1500, d=256, dtype="bf16", n_b=4, n_c=3,
                                      n_ec=2, n_r=3, k=8),
    "d64_long_windows": W("w4", N=1000, C=20000, d=64, dtype="bf16", n_b=64, n_c=16, n_ec=1,
                          n_r=2, k=8, target_alpha=1.0),
    "d192_small_batch": W("w5", N=97, C=999, d=192, dtype="bf16", n_b=8, n_c=4, n_ec=1, n_r=2,
                          k=8),
}


def run_window_gpu(w, X, Y, t, B, dloss=1.0, extra_flags=0):
    plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype,
                    flags=_lib.FLAG_ALL_NEGATIVES | extra_flags)
    assert plan.paths & _lib.PATH_ALL_NEGATIVES
    Xd, Yd, Bd = to_dev(X, w.dtype), to_dev(Y, w.dtype), to_dev(B, w.dtype)
    td = torch.from_numpy(t).cuda()
    ws = plan.workspace()
    ops.bucketize_sort(plan, Bd, Xd, Yd, ws)
    bx, by = (a.cpu().numpy() for a in plan.bucket_ids(ws))
    px, py = (a.cpu().numpy() for a in plan.permutations(ws))
    loss, row, sel, lse, _ = ops.loss_fwd(plan, Xd, Yd, td, ws)
    dl = torch.tensor([dloss], dtype=torch.float32, device="cuda")
    dX, dY = ops.loss_bwd(plan, Xd, Yd, td, sel, lse, dl, ws)
    return dict(bx=bx, by=by, px=px, py=py, loss=float(loss.item()), row=row.cpu().numpy(),
                lse=lse.cpu().numpy(), sel=sel.cpu().numpy(), dX=dX.cpu().numpy(),
                dY=dY.cpu().numpy(), status=ops.device_status(ws), paths=plan.paths)


def check_orders(g, n_r):
    for r in range(n_r):
        np.testing.assert_array_equal(g["px"][r], np.argsort(g["bx"][r], kind="stable"))
        np.testing.assert_array_equal(g["py"][r], np.argsort(g["by"][r], kind="stable"))


@pytest.mark.parametrize("name", sorted(CASES))
def test_window_parity(name):
    w = CASES[name]
    X, Y, t = synth.make_inputs(w, seed=5)
    B = synth.projections(5, 0, w.n_r, w.n_b, w.d, "bf16")
    g = run_window_gpu(w, X, Y, t, B, dloss=1.5)
    assert g["status"] == 0
    check_orders(g, w.n_r)
    o_loss, o_row, o_lse = oracle.window_loss(X, Y, t, g["px"], g["py"], w.n_c, w.n_ec)
    assert max_rel(g["row"], o_row) <= 1e-4
    assert max_rel(g["lse"], o_lse) <= 1e-4
    assert abs(g["loss"] - o_loss) <= 1e-4 * abs(o_loss)
    oX, oY = oracle.window_grad(X, Y, t, g["px"], g["py"], w.n_c, w.n_ec, o_lse, 1.5)
    assert max_rel(g["dX"], oX) <= 1e-3
    assert max_rel(g["dY"], oY) <= 1e-3
    assert np.all(g["sel"] == -1)


def test_window_exact_orders_on_integer_inputs():
    """Integer inputs: bucketing is exact, so the GPU's orders are the oracle's own."""
    w = W("wi", N=640, C=2500, d=64, dtype="bf16", n_b=16, n_c=5, n_ec=1, n_r=2, k=8)
    X, Y, t = synth.integer_inputs(w.N, w.C, w.d, lo=-2, hi=2, seed=4, scale=0.125)
    B = synth.integer_inputs(w.n_r * w.n_b, 1, w.d, lo=-2, hi=2, seed=9, scale=1.0)[0]
    B = B.reshape(w.n_r, w.n_b, w.d)
    g = run_window_gpu(w, X, Y, t, B)
    full = oracle.rece_forward(X, Y, t, B, w.n_c, w.n_ec, 1)
    np.testing.assert_array_equal(g["px"], full["permX"])
    np.testing.assert_array_equal(g["py"], full["permY"])
    _, o_row, o_lse = oracle.window_loss(X, Y, t, full["permX"], full["permY"], w.n_c, w.n_ec)
    assert max_rel(g["row"], o_row) <= 1e-4
    oX, oY = oracle.window_grad(X, Y, t, full["permX"], full["permY"], w.n_c, w.n_ec, o_lse)
    assert max_rel(g["dX"], oX) <= 1e-3 and max_rel(g["dY"], oY) <= 1e-3


def test_window_one_bucket_one_chunk_is_full_ce():
    w = W("wf", N=300, C=1000, d=64, dtype="bf16", n_b=1, n_c=1, n_ec=0, n_r=2, k=8)
    X, Y, t = synth.make_inputs(w, seed=6)
    B = synth.projections(6, 0, w.n_r, w.n_b, w.d, "bf16")
    g = run_window_gpu(w, X, Y, t, B)
    f_loss, f_row, f_lse = oracle.full_ce_loss(X, Y, t)
    assert max_rel(g["row"], f_row) <= 1e-4
    fX, fY = oracle.full_ce_grad(X, Y, t, f_lse)
    assert max_rel(g["dX"], fX) <= 1e-3 and max_rel(g["dY"], fY) <= 1e-3


def test_window_identical_rounds_and_determinism():
    """Three identical rounds count every pair three times, each copy weighted 1/3: the
    same loss and gradients as one round.  Two runs agree bit for bit."""
    w1 = W("w1r", N=600, C=4000, d=128, dtype="bf16", n_b=32, n_c=6, n_ec=1, n_r=1, k=8)
    w3 = W("w3r", N=600, C=4000, d=128, dtype="bf16", n_b=32, n_c=6, n_ec=1, n_r=3, k=8)
    X, Y, t = synth.make_inputs(w1, seed=8)
    B1 = synth.projections(8, 0, 1, w1.n_b, w1.d, "bf16")
    B3 = np.repeat(B1, 3, 0)
    a = run_window_gpu(w1, X, Y, t, B1)
    b = run_window_gpu(w3, X, Y, t, B3)
    c = run_window_gpu(w3, X, Y, t, B3)
    assert max_rel(b["row"], a["row"]) <= 1e-5
    assert max_rel(b["dX"], a["dX"]) <= 1e-4 and max_rel(b["dY"], a["dY"]) <= 1e-4
    for key in ("row", "lse", "dX", "dY"):
        assert np.array_equal(b[key], c[key]), key


# ---------------------------------------------------------------- on the CUDA cores
# fp32 exact mode, bf16 with RECE_FLAG_FMA_SCORES and bf16 widths the tcgen05 window
# kernels do not take: every score is the fixed-order fmaf chain, so the orders are the
# oracle's bit for bit (fmaf bucketing) and every value is within 1e-4 of its fp64 sums.
FMA_CASES = {
    "fp32_d64_rounds2": W("f1", N=600, C=3000, d=64, dtype="fp32", n_b=16, n_c=6, n_ec=1,
                          n_r=2, k=8),
    "fp32_d48_rounds3_ragged": W("f2", N=333, C=2001, d=48, dtype="fp32", n_b=7, n_c=5,
                                 n_ec=2, n_r=3, k=8, target_alpha=1.0),
    "fp32_d7_no_neighbours": W("f3", N=200, C=999, d=7, dtype="fp32", n_b=5, n_c=4, n_ec=0,
                               n_r=1, k=8),
    "bf16_fma_flag_d128": W("f4", N=500, C=2500, d=128, dtype="bf16", n_b=16, n_c=5, n_ec=1,
                            n_r=2, k=8),
}


@pytest.mark.parametrize("name", sorted(FMA_CASES))
def test_window_fma_parity(name):
    w = FMA_CASES[name]
    X, Y, t = synth.make_inputs(w, seed=12)
    B = synth.projections(12, 0, w.n_r, w.n_b, w.d, w.dtype)
    extra = _lib.FLAG_FMA_SCORES if w.dtype == "bf16" else 0
    g = run_window_gpu(w, X, Y, t, B, dloss=0.75, extra_flags=extra)
    assert g["paths"] & _lib.PATH_WINDOW_FMA
    assert g["status"] == 0
    full = oracle.rece_forward(X, Y, t, B, w.n_c, w.n_ec, 1)  # the oracle's own orders
    np.testing.assert_array_equal(g["bx"], full["bx"])
    np.testing.assert_array_equal(g["by"], full["by"])
    np.testing.assert_array_equal(g["px"], full["permX"])
    np.testing.assert_array_equal(g["py"], full["permY"])
    o_loss, o_row, o_lse = oracle.window_loss(X, Y, t, full["permX"], full["permY"], w.n_c,
                                              w.n_ec)
    assert max_rel(g["row"], o_row) <= 1e-4 and max_rel(g["lse"], o_lse) <= 1e-4
    assert abs(g["loss"] - o_loss) <= 1e-4 * abs(o_loss)
    oX, oY = oracle.window_grad(X, Y, t, full["permX"], full["permY"], w.n_c, w.n_ec, o_lse,
                                0.75)
    assert max_rel(g["dX"], oX) <= 1e-4 and max_rel(g["dY"], oY) <= 1e-4
    assert np.all(g["sel"] == -1)


def test_window_fma_wide_rows_and_determinism():
    """bf16 at d = 1024 (past the tcgen05 window kernels): bucketing on tcgen05, the window
    sums on the CUDA cores; the oracle on the GPU's orders, values within 1e-4; two runs
    agree bit for bit."""
    w = W("fw", N=256, C=1500, d=1024, dtype="bf16", n_b=16, n_c=3, n_ec=1, n_r=2, k=8)
    X, Y, t = synth.make_inputs(w, seed=13)
    B = synth.projections(13, 0, w.n_r, w.n_b, w.d, w.dtype)
    g = run_window_gpu(w, X, Y, t, B)
    assert g["paths"] & _lib.PATH_WINDOW_FMA and g["status"] == 0
    check_orders(g, w.n_r)
    _, o_row, o_lse = oracle.window_loss(X, Y, t, g["px"], g["py"], w.n_c, w.n_ec)
    assert max_rel(g["row"], o_row) <= 1e-4
    oX, oY = oracle.window_grad(X, Y, t, g["px"], g["py"], w.n_c, w.n_ec, o_lse)
    assert max_rel(g["dX"], oX) <= 1e-4 and max_rel(g["dY"], oY) <= 1e-4
    h = run_window_gpu(w, X, Y, t, B)
    for key in ("row", "lse", "dX", "dY"):
        assert np.array_equal(g[key], h[key]), key


def test_window_fma_one_bucket_one_chunk_is_full_ce():
    """fp32, n_b = n_c = 1: every item is in every row's window, once per round: the full
    cross-entropy (equation 3) and its gradient (equation 4), within 1e-4."""
    w = W("ff", N=200, C=700, d=32, dtype="fp32", n_b=1, n_c=1, n_ec=0, n_r=2, k=8)
    X, Y, t = synth.make_inputs(w, seed=14)
    B = synth.projections(14, 0, w.n_r, w.n_b, w.d)
    g = run_window_gpu(w, X, Y, t, B)
    f_loss, f_row, f_lse = oracle.full_ce_loss(X, Y, t)
    assert max_rel(g["row"], f_row) <= 1e-4
    fX, fY = oracle.full_ce_grad(X, Y, t, f_lse)
    assert max_rel(g["dX"], fX) <= 1e-4 and max_rel(g["dY"], fY) <= 1e-4
