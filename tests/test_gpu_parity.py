"""Parity of the CUDA path (through the C ABI) with the CPU oracle, element by element.

Bar: bucket ids, sort orders and selected index sets bit-exact (fmaf-chain scoring:
fp32 mode, and bf16 mode with RECE_FLAG_FMA_SCORES); loss, per-row loss, lse, dX and
dY within 1e-4 relative (max-norm), the oracle computing them in fp64.
"""
import numpy as np
import pytest
import torch

import oracle
from reduced_cross_entropy_b200 import ops, synth
from tests.gpu_common import max_rel, run_gpu, run_oracle, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-4
W = synth.WORKLOADS

CASES = {
    "tiny": W["tiny"],
    "tiny_bf16_rounds2": W["tiny"].scaled(256, 4096, dtype="bf16", n_r=2, k=40),
    "ragged": synth.Workload("ragged", N=1000, C=5003, d=48, dtype="fp32", n_b=37, n_c=13,
                             n_ec=2, n_r=3, k=50),
    "k_over_window": synth.Workload("kw", N=300, C=700, d=16, dtype="fp32", n_b=5, n_c=10,
                                    n_ec=0, n_r=2, k=200),
    "d_not_mult8": synth.Workload("d7", N=200, C=999, d=7, dtype="fp32", n_b=3, n_c=4, n_ec=1,
                                  n_r=1, k=20),
    "sasrec_scaled": W["sasrec"].scaled(3200, 12500, n_c=8),
    "lm_scaled": W["lm"].scaled(512, 4000, n_c=4, n_b=64, k=128, d=256),
    "large_norms_scaled": W["large"].scaled(2000, 20000, n_c=10, n_b=128, k=128),
    # C >= 2^18: the backward's pair sort takes three passes of at most 9-bit digits
    "three_pass_pair_sort": synth.Workload("p3", N=256, C=300001, d=16, dtype="fp32", n_b=8,
                                           n_c=16, n_ec=1, n_r=2, k=16),
    # wide rows: dY through the shared-memory ring of bulk row copies (d >= 1024)
    "lm_wide_fp32": W["lm"].scaled(384, 3000, n_c=3, n_b=32, k=64, d=2048, dtype="fp32"),
    "lm_wide_bf16": W["lm"].scaled(384, 3000, n_c=3, n_b=32, k=64, d=4096),
}


def compare(w, g, o, exact_indices=True):
    if exact_indices:
        np.testing.assert_array_equal(g["bx"], o["bx"])
        np.testing.assert_array_equal(g["by"], o["by"])
        np.testing.assert_array_equal(g["permX"], o["permX"])
        np.testing.assert_array_equal(g["permY"], o["permY"])
        np.testing.assert_array_equal(g["selected"], o["selected"])
    assert abs(g["loss"] - o["loss"]) <= TOL * abs(o["loss"])
    assert max_rel(g["row_loss"], o["row_loss"]) <= TOL
    assert max_rel(g["lse"], o["lse"]) <= TOL
    assert max_rel(g["dX"], o["dX"]) <= TOL
    assert max_rel(g["dY"], o["dY"]) <= TOL
    assert g["status"] == 0


@pytest.mark.parametrize("name", sorted(CASES))
def test_parity_fma_path(name):
    w = CASES[name]
    X, Y, t = synth.make_inputs(w, seed=0)
    B = synth.projections(0, 0, w.n_r, w.n_b, w.d, w.dtype)
    flags = 1 if w.dtype == "bf16" else 0
    compare(w, run_gpu(w, X, Y, t, B, flags=flags, dloss=0.75),
            run_oracle(w, X, Y, t, B, dloss=0.75))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_auto_bucket_plan_matches_oracle(dtype):
    """n_b = n_c = 0: the library takes the pages' n_b* at alpha_bc = 1 (RECE section 3,
    the paragraph before Algorithm 1): sqrt(4 * 3 * 600) = 84.9 -> n_b = n_c = 85 here; the
    path through that plan equals the oracle run at those values."""
    w = synth.Workload("auto", N=600, C=5000, d=64, dtype=dtype, n_b=85, n_c=85, n_ec=1,
                       n_r=2, k=40)
    X, Y, t = synth.make_inputs(w, seed=5)
    B = synth.projections(5, 0, w.n_r, w.n_b, w.d, w.dtype)
    g = run_gpu(w, X, Y, t, B, flags=1 if dtype == "bf16" else 0, auto_buckets=True)
    compare(w, g, run_oracle(w, X, Y, t, B))
    if dtype == "bf16":  # and on the tensor cores (tcgen05 sums: loss within 1e-2)
        o = run_oracle(w, X, Y, t, B)
        g = run_gpu(w, X, Y, t, B, auto_buckets=True)
        assert g["status"] & ~0x4 == 0
        assert abs(g["loss"] - o["loss"]) <= 1e-2 * abs(o["loss"])


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_draw_projections_match_oracle(dtype):
    """Algorithm 1's randn step drawn by the library (rece_draw_projections) against the
    oracle's draw of the same (seed, step) stream: the same fp32 numbers (one unit in the
    last place where the two sides' fp64 log / cos / sin differ at an fp32 rounding
    boundary, at most one element in 10^4), bf16 as the oracle's fp32 rounded to nearest
    even; then the fp32 path bucketized with the drawn vectors equals the oracle run."""
    w = synth.Workload("draw", N=700, C=4000, d=64, dtype=dtype, n_b=64, n_c=16, n_ec=1,
                       n_r=3, k=50)
    plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype)
    for seed, step in [(0, 0), (12345, 7), (2**63 + 5, 2**40)]:
        g = ops.draw_projections(plan, seed, step).float().cpu().numpy()
        o = oracle.draw_projections(seed, step, w.n_r, w.n_b, w.d)
        if dtype == "bf16":
            o = synth.round_bf16(o)
        diff = g != o
        assert diff.mean() <= 1e-4
        ulp = np.spacing(np.abs(o[diff])) * (2 ** 16 if dtype == "bf16" else 1)
        assert np.all(np.abs(g[diff] - o[diff]) <= ulp)
    if dtype == "fp32":
        X, Y, t = synth.make_inputs(w, seed=9)
        B = ops.draw_projections(plan, 9, 1).cpu().numpy()
        np.testing.assert_array_equal(B, oracle.draw_projections(9, 1, w.n_r, w.n_b, w.d))
        compare(w, run_gpu(w, X, Y, t, B), run_oracle(w, X, Y, t, B))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_autograd_wrapper_matches_the_calls_and_the_oracle(dtype):
    """ops.rece_loss (torch autograd over rece_loss_fwd / rece_loss_bwd, B drawn on the
    device from (seed, step)): the loss and the gradients torch hands back equal the direct
    calls' on the same B, and the oracle's within the mode's tolerance."""
    w = synth.Workload("autograd", N=700, C=5000, d=64, dtype=dtype, n_b=32, n_c=8, n_ec=1,
                       n_r=2, k=40)
    X, Y, t = synth.make_inputs(w, seed=3)
    plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype)
    Xd = to_dev(X, dtype).requires_grad_()
    Yd = to_dev(Y, dtype).requires_grad_()
    td = torch.from_numpy(t).cuda()
    loss = ops.rece_loss(Xd, Yd, td, (3, 5), plan)
    (0.5 * loss).backward()
    B = ops.draw_projections(plan, 3, 5)
    g = run_gpu(w, X, Y, t, B.float().cpu().numpy(), dloss=0.5)
    assert loss.item() == g["loss"]
    np.testing.assert_array_equal(Xd.grad.float().cpu().numpy(),
                                  torch.from_numpy(g["dX"]).to(Xd.dtype).float().numpy())
    np.testing.assert_array_equal(Yd.grad.float().cpu().numpy(),
                                  torch.from_numpy(g["dY"]).to(Yd.dtype).float().numpy())
    o = run_oracle(w, X, Y, t, B.float().cpu().numpy(), dloss=0.5)
    tol = 1e-4 if dtype == "fp32" else 1e-2
    assert abs(loss.item() - o["loss"]) <= tol * abs(o["loss"])


def test_fp32_exact_whole_arrays_at_sasrec_scale():
    """The fp32 exact mode at the SASRec-scale benchmark shape (N = 25,600, C = 100,000,
    n_b = 256, n_c = 64, n_ec = 1, n_r = 2, k = 256), the whole arrays against the whole
    oracle: bucket ids, orders and selected sets bit for bit, losses and gradients
    within 1e-4."""
    w = W["sasrec"].scaled(25_600, 100_000, dtype="fp32")
    X, Y, t = synth.make_inputs(w, seed=0)
    B = synth.projections(0, 0, w.n_r, w.n_b, w.d, w.dtype)
    compare(w, run_gpu(w, X, Y, t, B), run_oracle(w, X, Y, t, B))


def test_parity_ties_on_exact_inputs():
    """Integer-valued inputs: every score is exact and ties are everywhere, so the
    lowest-index tie rules of argmax, sort and selection are all exercised."""
    w = synth.Workload("ties", N=640, C=3000, d=12, dtype="fp32", n_b=6, n_c=16, n_ec=1,
                       n_r=2, k=37)
    X, Y, t = synth.integer_inputs(w.N, w.C, w.d, seed=3)
    B = synth.integer_inputs(w.n_r * w.n_b, 1, w.d, seed=4)[0].reshape(w.n_r, w.n_b, w.d)
    compare(w, run_gpu(w, X, Y, t, B), run_oracle(w, X, Y, t, B))


def test_full_ce_identity_one_bucket_one_chunk():
    """n_b = 1, n_c = 1, k = C - 1: the reduced loss is the full cross-entropy, and the
    fused full-CE op agrees with both."""
    w = synth.Workload("full", N=300, C=500, d=32, dtype="fp32", n_b=1, n_c=1, n_ec=0, n_r=1,
                       k=499)
    X, Y, t = synth.make_inputs(w, seed=7)
    B = synth.projections(7, 0, 1, 1, w.d)
    g = run_gpu(w, X, Y, t, B)
    o_loss, o_row, o_lse = oracle.full_ce_loss(X, Y, t)
    assert abs(g["loss"] - o_loss) <= TOL * o_loss
    assert max_rel(g["row_loss"], o_row) <= TOL
    Xd, Yd, td = to_dev(X, "fp32"), to_dev(Y, "fp32"), torch.from_numpy(t).cuda()
    loss, row, lse, ws = ops.full_ce_fwd(Xd, Yd, td)
    assert abs(loss.item() - o_loss) <= TOL * o_loss
    assert max_rel(row.cpu().numpy(), o_row) <= TOL
    dX, dY = ops.full_ce_bwd(Xd, Yd, td, lse, torch.ones(1, device="cuda"), ws)
    fX, fY = oracle.full_ce_grad(X, Y, t, o_lse)
    assert max_rel(dX.cpu().numpy(), fX) <= TOL
    assert max_rel(dY.cpu().numpy(), fY) <= TOL
    assert max_rel(g["dX"], fX) <= TOL and max_rel(g["dY"], fY) <= TOL


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_full_ce_op_parity(dtype):
    w = synth.Workload("fce", N=333, C=2049, d=40, dtype=dtype, n_b=1, n_c=1, n_ec=0, n_r=1,
                       k=1, target_alpha=1.0)
    X, Y, t = synth.make_inputs(w, seed=11)
    Xd, Yd, td = to_dev(X, dtype), to_dev(Y, dtype), torch.from_numpy(t).cuda()
    loss, row, lse, ws = ops.full_ce_fwd(Xd, Yd, td)
    o_loss, o_row, o_lse = oracle.full_ce_loss(X, Y, t)
    assert abs(loss.item() - o_loss) <= TOL * o_loss
    assert max_rel(row.cpu().numpy(), o_row) <= TOL
    assert max_rel(lse.cpu().numpy(), o_lse) <= TOL
    dX, dY = ops.full_ce_bwd(Xd, Yd, td, lse, torch.full((1,), 2.0, device="cuda"), ws)
    fX, fY = oracle.full_ce_grad(X, Y, t, o_lse, 2.0)
    assert max_rel(dX.cpu().numpy(), fX) <= TOL
    assert max_rel(dY.cpu().numpy(), fY) <= TOL


@pytest.mark.parametrize("N,C,d", [(333, 2049, 64), (200, 70_001, 64), (130, 3000, 256)])
def test_full_ce_op_on_tensor_cores(N, C, d):
    """bf16 with d a multiple of 64 up to 256: the fused exact full CE runs on tcgen05, as
    the all-negatives mode at one bucket, one chunk and one round (every item in every
    row's window, counted once; RECE equations 3 and 4).  Loss, row losses and lse within
    1e-4; gradients within 1e-3 (the probabilities reach the tensor cores as hi + lo
    bf16).  A catalogue past 2^16 items included."""
    w = synth.Workload("fce_tc", N=N, C=C, d=d, dtype="bf16", n_b=1, n_c=1, n_ec=0, n_r=1,
                       k=1, target_alpha=1.0)
    X, Y, t = synth.make_inputs(w, seed=21)
    Xd, Yd, td = to_dev(X, "bf16"), to_dev(Y, "bf16"), torch.from_numpy(t).cuda()
    assert ops.full_ce_workspace_bytes(N, C, d, "bf16") > ops.full_ce_workspace_bytes(N, C, 40,
                                                                                      "bf16")
    loss, row, lse, ws = ops.full_ce_fwd(Xd, Yd, td)
    o_loss, o_row, o_lse = oracle.full_ce_loss(X, Y, t)
    assert abs(loss.item() - o_loss) <= TOL * o_loss
    assert max_rel(row.cpu().numpy(), o_row) <= TOL
    assert max_rel(lse.cpu().numpy(), o_lse) <= TOL
    dX, dY = ops.full_ce_bwd(Xd, Yd, td, lse, torch.full((1,), 2.0, device="cuda"), ws)
    fX, fY = oracle.full_ce_grad(X, Y, t, o_lse, 2.0)
    assert max_rel(dX.cpu().numpy(), fX) <= 1e-3
    assert max_rel(dY.cpu().numpy(), fY) <= 1e-3
    assert ops.device_status(ws) == 0


def test_empty_batch():
    w = synth.Workload("empty", N=0, C=100, d=8, dtype="fp32", n_b=4, n_c=5, n_ec=1, n_r=1, k=3)
    X = np.zeros((0, 8), np.float32)
    Y = synth.make_inputs(w.scaled(5, 100), 0)[1]
    g = run_gpu(w, X, Y, np.zeros(0, np.int32), synth.projections(0, 0, 1, 4, 8))
    assert g["loss"] == 0.0
    assert g["dY"].shape == (100, 8) and np.all(g["dY"] == 0)


def test_single_item_catalogue():
    w = synth.Workload("one", N=50, C=1, d=8, dtype="fp32", n_b=2, n_c=1, n_ec=1, n_r=1, k=4)
    X, Y, _ = synth.make_inputs(w, 1)
    t = np.zeros(50, np.int32)
    g = run_gpu(w, X, Y, t, synth.projections(1, 0, 1, 2, 8))
    assert np.all(g["selected"] == -1)
    assert g["loss"] == 0.0 and np.all(g["row_loss"] == 0.0)
    assert np.all(g["dX"] == 0.0) and np.all(g["dY"] == 0.0)


def test_bad_target_sets_device_flag():
    w = W["tiny"].scaled(64, 512, n_c=4)
    X, Y, t = synth.make_inputs(w, 2)
    t[5] = w.C          # out of range
    t[9] = -3
    g = run_gpu(w, X, Y, t, synth.projections(2, 0, 1, w.n_b, w.d))
    assert g["status"] & 1
    assert np.isnan(g["row_loss"][5]) and np.isnan(g["row_loss"][9])
    ok = np.ones(64, bool)
    ok[[5, 9]] = False
    assert np.all(np.isfinite(g["row_loss"][ok]))


def test_backward_is_deterministic():
    w = CASES["sasrec_scaled"]
    X, Y, t = synth.make_inputs(w, seed=5)
    B = synth.projections(5, 0, w.n_r, w.n_b, w.d, w.dtype)
    a = run_gpu(w, X, Y, t, B, flags=1)
    b = run_gpu(w, X, Y, t, B, flags=1)
    for key in ("selected", "row_loss", "lse", "dX", "dY"):
        np.testing.assert_array_equal(a[key], b[key])
    assert a["loss"] == b["loss"]


def test_popular_items_summed_by_a_cta():
    """Items whose (item, row) runs exceed 256 pairs take the dY kernel that splits a run
    among a CTA's warps: here every row's positive is one of three items (runs of 300 to
    600 pairs and more) in the fp32 exact mode, against the oracle, and twice for
    determinism."""
    w = synth.Workload("popular", N=1200, C=2500, d=24, dtype="fp32", n_b=8, n_c=6, n_ec=1,
                       n_r=2, k=40)
    X, Y, _ = synth.make_inputs(w, seed=8)
    t = np.array([(0, 0, 7, 1999)[i % 4] for i in range(w.N)], dtype=np.int32)
    B = synth.projections(8, 0, w.n_r, w.n_b, w.d, w.dtype)
    g = run_gpu(w, X, Y, t, B, dloss=1.25)
    compare(w, g, run_oracle(w, X, Y, t, B, dloss=1.25))
    again = run_gpu(w, X, Y, t, B, dloss=1.25)
    np.testing.assert_array_equal(g["dY"], again["dY"])


def test_sort_many_buckets_and_one_bucket():
    for n_b in (4096, 1):
        w = synth.Workload("sort", N=20000, C=30011, d=16, dtype="fp32", n_b=n_b, n_c=16,
                           n_ec=1, n_r=1, k=8)
        X, Y, t = synth.make_inputs(w, 9)
        B = synth.projections(9, 0, 1, n_b, 16)
        plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode="fp32")
        ws = plan.workspace()
        ops.bucketize_sort(plan, to_dev(B, "fp32"), to_dev(X, "fp32"), to_dev(Y, "fp32"), ws)
        bx, by = (a.cpu().numpy()[0] for a in plan.bucket_ids(ws))
        px, py = (a.cpu().numpy()[0] for a in plan.permutations(ws))
        np.testing.assert_array_equal(bx, oracle.bucketize(X, B[0]))
        np.testing.assert_array_equal(by, oracle.bucketize(Y, B[0]))
        np.testing.assert_array_equal(px, np.argsort(bx, kind="stable"))
        np.testing.assert_array_equal(py, np.argsort(by, kind="stable"))
        starts = plan.bucket_starts_y(ws).cpu().numpy()[0]
        np.testing.assert_array_equal(starts[:n_b + 1],
                                      np.searchsorted(np.sort(by), np.arange(n_b + 1)))


@pytest.mark.parametrize("name", ["ragged", "sasrec_scaled", "d_not_mult8"])
def test_logits_output_and_both_backward_paths(name):
    """rece_loss_fwd's logits are the positive's and the selected items' logits; the
    backward gives the same gradients from them as when it recomputes them."""
    w = CASES[name]
    X, Y, t = synth.make_inputs(w, seed=1)
    B = synth.projections(1, 0, w.n_r, w.n_b, w.d, w.dtype)
    flags = 1 if w.dtype == "bf16" else 0
    a = run_gpu(w, X, Y, t, B, flags=flags, use_logits=True)
    b = run_gpu(w, X, Y, t, B, flags=flags, use_logits=False)
    o = run_oracle(w, X, Y, t, B)
    lg = a["logits"]
    sel = a["selected"]
    want = np.full_like(lg, -np.inf)
    X64, Y64 = X.astype(np.float64), Y.astype(np.float64)
    want[:, 0] = np.einsum("nd,nd->n", X64, Y64[t])
    for i in range(w.N):
        s = sel[i][sel[i] >= 0]
        want[i, 1:1 + len(s)] = Y64[s] @ X64[i]
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(lg), fin)
    assert np.abs(lg[fin] - want[fin]).max() <= 1e-5 * max(1.0, np.abs(want[fin]).max())
    for g in (a, b):
        assert max_rel(g["dX"], o["dX"]) <= TOL and max_rel(g["dY"], o["dY"]) <= TOL
    assert max_rel(a["dX"], b["dX"]) <= TOL and max_rel(a["dY"], b["dY"]) <= TOL
