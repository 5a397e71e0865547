"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each test below checks one oracle function against an independent source: a library
routine (numpy argmax / stable argsort, torch cross-entropy and autograd), brute force
on inputs whose arithmetic is exact in fp32 (so every summation order agrees), a
hand-worked example of the RECE paper's Algorithm 1 (tests/golden), closed forms,
finite differences, or invariants of the definition.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from reduced_cross_entropy_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- helpers
def brute_chunks(M, n_c):
    """Chunk membership straight from the set-builder definition, in exact rationals:
    element i is in chunk c when c*M/n_c <= i < (c+1)*M/n_c."""
    out = []
    for c in range(n_c):
        lo, hi = Fraction(c * M, n_c), Fraction((c + 1) * M, n_c)
        out.append([i for i in range(M) if lo <= i < hi])
    return out


def brute_forward(Xi, Yi, z, Bi, n_c, n_ec, k):
    """Independent brute force on integer-valued inputs (exact integer scores).

    Xi, Yi, Bi are integer arrays; scores are exact integer dot products.  Buckets by
    first-max argmax, stable sort by Python's sorted, chunks by exact rationals,
    windows as explicit unions of sets, candidates as a set, order by (-score, id)."""
    N, C = len(Xi), len(Yi)
    n_r = len(Bi)
    cand = [set() for _ in range(N)]
    for r in range(n_r):
        bx = [max(range(len(Bi[r])), key=lambda b: (int(np.dot(Bi[r][b], Xi[i])), -b))
              for i in range(N)]
        by = [max(range(len(Bi[r])), key=lambda b: (int(np.dot(Bi[r][b], Yi[j])), -b))
              for j in range(C)]
        px = sorted(range(N), key=lambda i: bx[i])
        py = sorted(range(C), key=lambda j: by[j])
        xch, ych = brute_chunks(N, n_c), brute_chunks(C, n_c)
        for c in range(n_c):
            window = set()
            for cc in range(c - n_ec, c + n_ec + 1):
                if 0 <= cc < n_c:
                    window |= {py[q] for q in ych[cc]}
            for p in xch[c]:
                i = px[p]
                cand[i] |= window - {int(z[i])}
    sel = np.full((N, k), -1, np.int64)
    for i in range(N):
        order = sorted(cand[i], key=lambda j: (-int(np.dot(Xi[i], Yi[j])), j))[:k]
        sel[i, :len(order)] = order
    return sel, [len(c) for c in cand]


def rel_err(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


# --------------------------------------------------------------------------- golden
def test_golden_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_alg1.json")))
    X, Y = np.array(g["X"], np.float32), np.array(g["Y"], np.float32)
    B = np.array(g["B"], np.float32)
    t = np.array(g["targets"], np.int32)
    for case in g["cases"]:
        out = oracle.rece_forward(X, Y, t, B, g["n_c"], g["n_ec"], case["k"])
        assert out["bx"].tolist() == g["bx"]
        assert out["by"].tolist() == g["by"]
        assert out["permX"].tolist() == g["permX"]
        assert out["permY"].tolist() == g["permY"]
        assert out["selected"].tolist() == case["selected"]
        want = [eval(e, {"log": math.log, "e": math.e}) for e in case["row_loss_expr"]]
        np.testing.assert_allclose(out["row_loss"], want, rtol=1e-14)
        assert out["loss"] == pytest.approx(sum(want) / 4, rel=1e-14)


# --------------------------------------------------------------------------- step 1
def test_bucketize_matches_numpy_argmax_on_exact_inputs():
    rng = np.random.default_rng(1)
    for d, n_b in [(1, 1), (3, 5), (8, 16), (17, 7)]:
        Vi = rng.integers(-3, 4, size=(200, d))
        Bi = rng.integers(-2, 3, size=(n_b, d))
        want = np.argmax(Vi @ Bi.T, axis=1)          # first maximum -> lowest b
        got = oracle.bucketize(Vi.astype(np.float32) * 0.5, Bi.astype(np.float32))
        np.testing.assert_array_equal(got, want)


def test_bucketize_invariants():
    rng = np.random.default_rng(2)
    V = rng.standard_normal((300, 24)).astype(np.float32)
    B = rng.standard_normal((9, 24)).astype(np.float32)
    assert np.all(oracle.bucketize(V, B[:1]) == 0)                       # n_b = 1
    np.testing.assert_array_equal(oracle.bucketize(V * 2, B), oracle.bucketize(V, B))
    Bdup = np.concatenate([B[:3], B[:3]])                                # planted ties
    assert np.all(oracle.bucketize(V, Bdup) < 3)


# --------------------------------------------------------------------------- step 2
def test_stable_argsort_matches_numpy():
    rng = np.random.default_rng(3)
    for M, nk in [(1, 1), (10, 1), (1000, 7), (5000, 256)]:
        keys = rng.integers(0, nk, size=M).astype(np.int32)
        np.testing.assert_array_equal(oracle.stable_argsort(keys),
                                      np.argsort(keys, kind="stable"))


# --------------------------------------------------------------------------- step 3
@pytest.mark.parametrize("M,n_c", [(10, 3), (7, 7), (100, 64), (4096, 8), (33, 1)])
def test_chunk_starts_match_set_builder(M, n_c):
    ch = brute_chunks(M, n_c)
    for c in range(n_c):
        assert oracle.chunk_start(c, M, n_c) == ch[c][0]
    assert oracle.chunk_start(n_c, M, n_c) == M


def test_chunk_sizes_closed_form():
    for w in synth.WORKLOADS.values():
        for M in (w.N, w.C):
            sizes = [oracle.chunk_start(c + 1, M, w.n_c) - oracle.chunk_start(c, M, w.n_c)
                     for c in range(w.n_c)]
            assert sum(sizes) == M
            assert max(sizes) - min(sizes) <= 1
            assert set(sizes) <= {M // w.n_c, -(-M // w.n_c)}
    w = synth.WORKLOADS["sasrec"]
    ys = {oracle.chunk_start(c + 1, w.C, 64) - oracle.chunk_start(c, w.C, 64) for c in range(64)}
    assert ys == {1562, 1563}


# --------------------------------------------------------------------------- step 4
@pytest.mark.parametrize("N,C,d,n_b,n_c,n_ec,n_r,k", [
    (12, 40, 4, 3, 3, 1, 1, 5),
    (16, 64, 3, 4, 4, 0, 2, 8),
    (9, 30, 5, 2, 5, 2, 2, 40),     # k above every candidate count
    (8, 8, 2, 1, 1, 0, 1, 7),       # one bucket, one chunk: full catalogue
    (15, 50, 6, 5, 7, 1, 3, 3),
])
def test_selection_brute_force_exact_inputs(N, C, d, n_b, n_c, n_ec, n_r, k):
    rng = np.random.default_rng(N * 1000 + C)
    Xi = rng.integers(-2, 3, size=(N, d))
    Yi = rng.integers(-2, 3, size=(C, d))
    Bi = rng.integers(-2, 3, size=(n_r, n_b, d))
    z = rng.integers(0, C, size=N).astype(np.int32)
    want, ncand = brute_forward(Xi, Yi, z, Bi, n_c, n_ec, k)
    out = oracle.rece_forward(Xi.astype(np.float32) * 0.25, Yi.astype(np.float32) * 0.5, z,
                              Bi.astype(np.float32), n_c, n_ec, k)
    np.testing.assert_array_equal(out["selected"], want)
    np.testing.assert_array_equal(out["n_cand"], ncand)


def _random_case(N=64, C=300, d=16, n_b=4, n_c=4, n_r=2, seed=5):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((N, d)) / 4).astype(np.float32)
    Y = (rng.standard_normal((C, d)) / 4).astype(np.float32)
    B = rng.standard_normal((n_r, n_b, d)).astype(np.float32)
    z = rng.integers(0, C, size=N).astype(np.int32)
    return X, Y, z, B


def test_selection_properties_random_inputs():
    X, Y, z, B = _random_case()
    n_c, n_ec = 4, 1
    outs = {k: oracle.rece_forward(X, Y, z, B, n_c, n_ec, k) for k in (1, 5, 20, 400)}
    full = outs[400]
    N, C = len(X), len(Y)
    for i in range(N):
        # candidates rebuilt from the oracle's own orders, with the chunk starts
        cand = set()
        for r in range(B.shape[0]):
            p = int(np.nonzero(full["permX"][r] == i)[0][0])
            c = max(cc for cc in range(n_c) if oracle.chunk_start(cc, N, n_c) <= p)
            lo = oracle.chunk_start(max(0, c - n_ec), C, n_c)
            hi = oracle.chunk_start(min(n_c, c + n_ec + 1), C, n_c)
            cand |= set(full["permY"][r][lo:hi].tolist())
        cand.discard(int(z[i]))
        # k >= candidate count -> the selection is the whole window minus the positive
        assert set(full["selected"][i][full["selected"][i] >= 0].tolist()) == cand
        for k in (1, 5, 20):
            s = outs[k]["selected"][i]
            s = s[s >= 0]
            assert list(s) == list(full["selected"][i][:len(s)])        # nested prefixes
            scores = {j: oracle.dot_f32(X[i], Y[j]) for j in cand}
            rest = cand - set(s.tolist())
            if len(s) and rest:
                assert min(scores[j] for j in s) >= max(scores[j] for j in rest)
    # monotone in k, bounded by full CE, nonnegative
    _, fce_row, _ = oracle.full_ce_loss(X, Y, z)
    prev = np.zeros(N)
    for k in (1, 5, 20, 400):
        row = outs[k]["row_loss"]
        assert np.all(row >= prev - 1e-12)
        assert np.all(row <= fce_row + 1e-12)
        prev = row
    assert np.all(outs[1]["row_loss"] > 0)


def test_identical_rounds_equal_one_round():
    X, Y, z, B = _random_case(n_r=1)
    one = oracle.rece_forward(X, Y, z, B, 4, 1, 17)
    two = oracle.rece_forward(X, Y, z, np.concatenate([B, B]), 4, 1, 17)
    np.testing.assert_array_equal(one["selected"], two["selected"])
    assert one["loss"] == two["loss"]


# --------------------------------------------------------------------------- step 5
def test_full_ce_matches_torch():
    X, Y, z, _ = _random_case(N=40, C=120, d=12)
    loss, row, lse = oracle.full_ce_loss(X, Y, z)
    logits = torch.from_numpy(X).double() @ torch.from_numpy(Y).double().T
    ref = torch.nn.functional.cross_entropy(logits, torch.from_numpy(z).long(),
                                            reduction="none")
    np.testing.assert_allclose(row, ref.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, 1).numpy(), rtol=1e-13)
    assert loss == pytest.approx(float(ref.mean()), rel=1e-12)


@pytest.mark.parametrize("n_ec", [0, 1, 3])
def test_reduced_equals_full_ce_one_bucket_one_chunk(n_ec):
    """n_b = 1, n_c = 1, k = C - 1: the window is the catalogue, so the reduced loss is
    the full cross-entropy of equation (3)."""
    X, Y, z, B = _random_case(N=30, C=90, d=8, n_b=1, n_r=1)
    out = oracle.rece_forward(X, Y, z, B, 1, n_ec, len(Y) - 1)
    loss, row, lse = oracle.full_ce_loss(X, Y, z)
    assert np.all(out["n_cand"] == len(Y) - 1)
    np.testing.assert_allclose(out["row_loss"], row, rtol=1e-12)
    np.testing.assert_allclose(out["lse"], lse, rtol=1e-13)
    assert out["loss"] == pytest.approx(loss, rel=1e-12)


def test_empty_candidates_and_empty_batch():
    # C = 1: the only item is every row's positive -> no negatives, loss 0
    X = np.ones((3, 4), np.float32)
    Y = np.ones((1, 4), np.float32)
    out = oracle.rece_forward(X, Y, np.zeros(3, np.int32), np.ones((1, 2, 4), np.float32),
                              1, 1, 4)
    assert np.all(out["selected"] == -1)
    assert out["loss"] == 0.0
    loss, row, lse = oracle.rece_loss(np.zeros((0, 4), np.float32), Y, np.zeros(0, np.int32),
                                      np.zeros((0, 2), np.int32))
    assert loss == 0.0 and row.shape == (0,)


# --------------------------------------------------------------------------- step 6
def _dyadic_case(N=6, C=24, d=4, seed=11):
    """Inputs on a 2^-12 grid so that x +- 2^-10 is exact in fp32."""
    rng = np.random.default_rng(seed)
    X = rng.integers(-1500, 1500, size=(N, d)).astype(np.float32) / 4096
    Y = rng.integers(-1500, 1500, size=(C, d)).astype(np.float32) / 4096
    B = rng.standard_normal((2, 3, d)).astype(np.float32)
    z = rng.integers(0, C, size=N).astype(np.int32)
    return X, Y, z, B


def test_rece_grad_finite_differences():
    X, Y, z, B = _dyadic_case()
    n_c, n_ec, k = 2, 0, 3
    base = oracle.rece_forward(X, Y, z, B, n_c, n_ec, k)
    sel = base["selected"]
    dloss = 0.7
    dX, dY = oracle.rece_grad(X, Y, z, sel, base["lse"], dloss)
    h = 2.0 ** -10
    checked = 0
    for name, A, G in (("X", X, dX), ("Y", Y, dY)):
        for idx in np.ndindex(A.shape):
            losses = []
            for s in (+1, -1):
                P = A.copy()
                P[idx] = P[idx] + np.float32(s * h)
                XX, YY = (P, Y) if name == "X" else (X, P)
                again = oracle.rece_forward(XX, YY, z, B, n_c, n_ec, k)
                if not np.array_equal(again["selected"], sel):
                    losses = None          # selection changed: not differentiable here
                    break
                losses.append(oracle.rece_loss(XX, YY, z, sel)[0])
            if losses is None:
                continue
            fd = dloss * (losses[0] - losses[1]) / (2 * h)
            assert fd == pytest.approx(G[idx], abs=1e-6 * max(1.0, np.abs(G).max()))
            checked += 1
    assert checked > 0.8 * (X.size + Y.size)


def test_rece_grad_invariants():
    X, Y, z, B = _random_case(N=50, C=400, d=8)
    out = oracle.rece_forward(X, Y, z, B, 8, 0, 6)
    dX, dY = oracle.rece_grad(X, Y, z, out["selected"], out["lse"], 1.0)
    # every row's coefficients sum to zero -> the dY rows sum to the zero vector
    assert np.abs(dY.sum(0)).max() < 1e-12
    touched = set(z.tolist()) | set(out["selected"][out["selected"] >= 0].tolist())
    untouched = sorted(set(range(len(Y))) - touched)
    assert len(untouched) > 0 and np.all(dY[untouched] == 0.0)


def test_rece_grad_row_and_item_samples_match_the_full_gradient():
    """rece_grad_rows / rece_grad_items (the full-size parity checks' expected values)
    against rece_grad, which finite differences and autograd pin; a planted duplicate entry
    and an item nobody selects cover the counting rules."""
    X, Y, z, B = _random_case(N=60, C=300, d=8)
    out = oracle.rece_forward(X, Y, z, B, 6, 1, 5)
    sel, lse = out["selected"].copy(), out["lse"]
    sel[3, 0] = sel[3, 1]  # a duplicate entry counts twice, as rece_grad counts it
    _, _, lse = oracle.rece_loss(X, Y, z, sel)
    dX, dY = oracle.rece_grad(X, Y, z, sel, lse, 0.7)
    rows = np.array([0, 3, 17, 59])
    gX = oracle.rece_grad_rows(X, Y, z, rows, sel[rows], lse[rows], 0.7)
    assert rel_err(gX, dX[rows]) < 1e-12
    touched = set(z.tolist()) | set(sel[sel >= 0].tolist())
    nobody = min(set(range(len(Y))) - touched)
    items = [int(z[0]), int(sel[3, 1]), int(sel[10, 2]), nobody, len(Y) - 1]
    every = np.arange(len(X))
    gY = oracle.rece_grad_items(X, Y, z, every, sel, lse, items, 0.7)
    assert rel_err(gY, dY[items]) < 1e-12
    assert np.all(gY[3] == 0.0)
    # rows that hold none of the items may be left out
    keep = np.nonzero(np.isin(sel, items).any(axis=1) | np.isin(z, items))[0]
    assert len(keep) < len(X)
    gY2 = oracle.rece_grad_items(X, Y, z, keep, sel[keep], lse[keep], items, 0.7)
    assert rel_err(gY2, dY[items]) < 1e-12


def test_rece_grad_equals_full_ce_grad_in_full_case():
    X, Y, z, B = _random_case(N=20, C=50, d=6, n_b=1, n_r=1)
    out = oracle.rece_forward(X, Y, z, B, 1, 0, len(Y) - 1)
    dX, dY = oracle.rece_grad(X, Y, z, out["selected"], out["lse"], 1.3)
    _, _, lse = oracle.full_ce_loss(X, Y, z)
    fX, fY = oracle.full_ce_grad(X, Y, z, lse, 1.3)
    assert rel_err(dX, fX) < 1e-12 and rel_err(dY, fY) < 1e-12


def test_full_ce_grad_matches_torch_autograd():
    X, Y, z, _ = _random_case(N=16, C=70, d=5)
    _, _, lse = oracle.full_ce_loss(X, Y, z)
    dX, dY = oracle.full_ce_grad(X, Y, z, lse, 2.0)
    Xt = torch.from_numpy(X).double().requires_grad_()
    Yt = torch.from_numpy(Y).double().requires_grad_()
    loss = 2.0 * torch.nn.functional.cross_entropy(Xt @ Yt.T, torch.from_numpy(z).long())
    loss.backward()
    assert rel_err(dX, Xt.grad.numpy()) < 1e-12
    assert rel_err(dY, Yt.grad.numpy()) < 1e-12


# --------------------------------------------------------------------------- sampled baselines
def _sampled_case(N=24, C=60, d=7, n=9, seed=5, pad=True):
    X, Y, z, _ = _random_case(N=N, C=C, d=d)
    rng = np.random.default_rng(seed)
    neg = rng.integers(0, C, size=(N, n)).astype(np.int32)
    neg[0, :] = z[0]                      # the positive sampled as a negative
    neg[1, 1] = neg[1, 0]                 # a negative drawn twice
    if pad:
        neg[2, -3:] = -1                  # padding
    return X, Y, z, neg


def _torch_sampled_rows(kind, X, Y, z, neg):
    """Row losses from torch's own loss routines on the [positive, negatives] logits."""
    Xt, Yt = torch.from_numpy(X).double(), torch.from_numpy(Y).double()
    rows = []
    for i in range(len(X)):
        js = [int(z[i])] + [int(j) for j in neg[i] if j >= 0]
        lg = Xt[i] @ Yt[js].T
        if kind == oracle.SAMPLED_CE_MINUS:
            rows.append(torch.nn.functional.cross_entropy(lg[None], torch.zeros(1).long()))
        else:
            lab = torch.zeros_like(lg)
            lab[0] = 1.0
            rows.append(torch.nn.functional.binary_cross_entropy_with_logits(
                lg, lab, reduction="sum"))
    return torch.stack(rows) if rows else torch.zeros(0, dtype=torch.float64)


@pytest.mark.parametrize("kind", [0, 1])
def test_sampled_loss_matches_torch_losses(kind):
    """Equation (2) is torch's cross-entropy over [l+, l_neg...] with class 0; equation
    (1) is torch's BCE-with-logits with label 1 on l+ and 0 on every sampled negative."""
    X, Y, z, neg = _sampled_case()
    loss, row, lse = oracle.sampled_loss(kind, X, Y, z, neg)
    ref = _torch_sampled_rows(kind, X, Y, z, neg).numpy()
    np.testing.assert_allclose(row, ref, rtol=1e-12, atol=1e-12)
    assert loss == pytest.approx(float(ref.mean()), rel=1e-12)


def test_bce_plus_far_tails_stay_finite():
    """Logits of +-800: -log sigmoid(800) ~ 0 and -log(1 - sigmoid(800)) = 800 + ~0,
    where a naive log(1 + exp(l)) overflows."""
    X = np.array([[1.0]], np.float32)
    Y = np.array([[800.0], [-800.0]], np.float32)
    loss, row, _ = oracle.sampled_loss(1, X, Y, np.array([0], np.int32),
                                       np.array([[0, 1, 0]], np.int32))
    assert row[0] == pytest.approx(2 * 800.0, rel=1e-15)


def test_ce_minus_over_the_rest_of_the_catalogue_is_full_ce():
    """Every item but the positive sampled once: equation (2) is equation (3)."""
    X, Y, z, _ = _random_case(N=20, C=40, d=6)
    neg = np.array([[j for j in range(len(Y)) if j != z[i]] for i in range(len(X))],
                   np.int32)
    loss, row, lse = oracle.sampled_loss(0, X, Y, z, neg)
    floss, frow, flse = oracle.full_ce_loss(X, Y, z)
    np.testing.assert_allclose(row, frow, rtol=1e-12)
    np.testing.assert_allclose(lse, flse, rtol=1e-13)
    dX, dY = oracle.sampled_grad(0, X, Y, z, neg, lse, 0.9)
    fX, fY = oracle.full_ce_grad(X, Y, z, flse, 0.9)
    assert rel_err(dX, fX) < 1e-12 and rel_err(dY, fY) < 1e-12


@pytest.mark.parametrize("kind", [0, 1])
def test_sampled_grad_matches_torch_autograd(kind):
    X, Y, z, neg = _sampled_case(N=12, C=30, d=5, n=6)
    _, _, lse = oracle.sampled_loss(kind, X, Y, z, neg)
    dX, dY = oracle.sampled_grad(kind, X, Y, z, neg, lse, 1.7)
    Xt = torch.from_numpy(X).double().requires_grad_()
    Yt = torch.from_numpy(Y).double().requires_grad_()
    rows = []
    for i in range(len(X)):
        js = [int(z[i])] + [int(j) for j in neg[i] if j >= 0]
        lg = Xt[i] @ Yt[js].T
        if kind == 0:
            rows.append(torch.logsumexp(lg, 0) - lg[0])
        else:
            rows.append(-torch.nn.functional.logsigmoid(lg[0])
                        - torch.nn.functional.logsigmoid(-lg[1:]).sum())
    (1.7 * torch.stack(rows).mean()).backward()
    assert rel_err(dX, Xt.grad.numpy()) < 1e-12
    assert rel_err(dY, Yt.grad.numpy()) < 1e-12


@pytest.mark.parametrize("kind", [0, 1])
def test_sampled_grad_finite_differences(kind):
    X, Y, z, _ = _dyadic_case(N=5, C=12, d=3)
    neg = np.random.default_rng(3).integers(0, 12, size=(5, 4)).astype(np.int32)
    _, _, lse = oracle.sampled_loss(kind, X, Y, z, neg)
    dloss = 0.6
    dX, dY = oracle.sampled_grad(kind, X, Y, z, neg, lse, dloss)
    h = 2.0 ** -10
    for name, A, G in (("X", X, dX), ("Y", Y, dY)):
        for idx in np.ndindex(A.shape):
            ls = []
            for sgn in (+1, -1):
                P = A.copy()
                P[idx] = P[idx] + np.float32(sgn * h)
                XX, YY = (P, Y) if name == "X" else (X, P)
                ls.append(oracle.sampled_loss(kind, XX, YY, z, neg)[0])
            fd = dloss * (ls[0] - ls[1]) / (2 * h)
            assert fd == pytest.approx(G[idx], abs=1e-6 * max(1.0, np.abs(G).max()))


def test_sampled_invariants():
    X, Y, z, neg = _sampled_case(pad=False)
    N = len(X)
    # padding takes no part
    padded = np.concatenate([neg, np.full((N, 4), -1, np.int32)], 1)
    for kind in (0, 1):
        assert np.array_equal(oracle.sampled_loss(kind, X, Y, z, neg)[1],
                              oracle.sampled_loss(kind, X, Y, z, padded)[1])
    # BCE+: the negatives' terms are independent, so the loss is additive over a split
    a, b = neg[:, :4], neg[:, 4:]
    none = np.zeros((N, 0), np.int32)
    r_ab = oracle.sampled_loss(1, X, Y, z, neg)[1]
    r_a = oracle.sampled_loss(1, X, Y, z, a)[1]
    r_b = oracle.sampled_loss(1, X, Y, z, b)[1]
    r_0 = oracle.sampled_loss(1, X, Y, z, none)[1]
    np.testing.assert_allclose(r_ab, r_a + r_b - r_0, rtol=1e-12)
    # CE- with no negatives: the softmax over the positive alone, loss exactly 0
    assert np.all(oracle.sampled_loss(0, X, Y, z, none)[1] == 0.0)
    # CE-: more negatives never lower a row's loss (the denominator only grows)
    assert np.all(oracle.sampled_loss(0, X, Y, z, a)[1] <=
                  oracle.sampled_loss(0, X, Y, z, neg)[1] + 1e-15)
    # every row's CE- coefficients sum to zero -> the dY rows sum to the zero vector
    _, _, lse = oracle.sampled_loss(0, X, Y, z, neg)
    _, dY = oracle.sampled_grad(0, X, Y, z, neg, lse, 1.0)
    assert np.abs(dY.sum(0)).max() < 1e-12


# --------------------------------------------------------------------------- inputs
def test_bf16_rounding_is_round_to_nearest_even():
    vals = np.array([1.0, 1.00390625, 1.005859375, 1.0078125 + 2 ** -9, -3.3, 0.0],
                    np.float32)
    want = torch.from_numpy(vals).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(synth.round_bf16(vals), want)
    rng = np.random.default_rng(0)
    v = rng.standard_normal(10000).astype(np.float32)
    np.testing.assert_array_equal(synth.round_bf16(v),
                                  torch.from_numpy(v).to(torch.bfloat16).float().numpy())


# --------------------------------------------------------------------------- memory model
def test_optimal_buckets_closed_forms():
    # 4 * 1 * (1 + 2) * 10000 = 120000 -> sqrt = 346.41 -> 346, n_c = 346 / 1 = 346
    assert oracle.optimal_buckets(10000, 10 ** 6, 1, 1.0) == (346, 346)
    # alpha_bc = 0.25, n_ec = 0, min = 2500: sqrt(2500) = 50, n_c = 200
    assert oracle.optimal_buckets(2500, 3000, 0, 0.25) == (50, 200)
    # the count is symmetric in N and C (min of the two), clamped at 4096
    assert oracle.optimal_buckets(7, 10 ** 9, 2, 2.0) == oracle.optimal_buckets(10 ** 9, 7, 2, 2.0)
    assert oracle.optimal_buckets(10 ** 9, 10 ** 9, 3, 4.0)[0] == 4096


def test_memory_model_matches_the_stated_ratio():
    """The pages state the model is sqrt(min) / (2 r sqrt(alpha_bc (1 + 2 n_ec))) times
    below the full cross-entropy's N * C logits; check that ratio on a grid."""
    for N, C, n_ec, n_r, a in [(25600, 100000, 1, 2, 4.0), (51200, 10 ** 6, 1, 2, 1.0),
                               (300, 200, 0, 1, 0.5), (16384, 128000, 2, 3, 2.0)]:
        model = oracle.memory_model_elements(N, C, n_ec, n_r, a)
        ratio = math.sqrt(min(N, C)) / (2 * n_r * math.sqrt(a * (1 + 2 * n_ec)))
        assert N * C / model == pytest.approx(ratio, rel=1e-12)
    # the minimised quantity: at alpha_bc = 1, n_ec = 0, r = 1, min = max = M: 2 M^1.5
    assert oracle.memory_model_elements(400, 400, 0, 1, 1.0) == pytest.approx(2 * 400 ** 1.5)


# --------------------------------------------------------------------------- Algorithm 1 as printed
@pytest.mark.parametrize("n_c,n_ec,n_r", [(4, 1, 2), (5, 0, 3), (3, 2, 1), (6, 1, 2)])
def test_window_loss_ln_count_equals_deduplicated_union(n_c, n_ec, n_r):
    """The rounds paragraph's ln(count) correction makes every duplicated pair count once:
    the literal loss equals the top-k path with k at least the number of candidates (the
    de-duplicated union), a separately written selection-based oracle."""
    X, Y, z, B = _random_case(N=48, C=120, d=8, n_b=3, n_c=n_c, n_r=n_r, seed=n_c + n_r)
    top = oracle.rece_forward(X, Y, z, B, n_c, n_ec, len(Y))
    assert np.all(top["n_cand"] <= len(Y))
    loss, row, lse = oracle.window_loss(X, Y, z, top["permX"], top["permY"], n_c, n_ec)
    np.testing.assert_allclose(row, top["row_loss"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, top["lse"], rtol=1e-13)
    dX, dY = oracle.window_grad(X, Y, z, top["permX"], top["permY"], n_c, n_ec, lse, 0.8)
    tX, tY = oracle.rece_grad(X, Y, z, top["selected"], top["lse"], 0.8)
    assert rel_err(dX, tX) < 1e-12 and rel_err(dY, tY) < 1e-12


def test_window_loss_one_bucket_one_chunk_is_full_ce():
    X, Y, z, B = _random_case(N=30, C=70, d=6, n_b=1, n_c=1, n_r=2)
    top = oracle.rece_forward(X, Y, z, B, 1, 0, 1)
    loss, row, lse = oracle.window_loss(X, Y, z, top["permX"], top["permY"], 1, 0)
    f_loss, f_row, f_lse = oracle.full_ce_loss(X, Y, z)
    np.testing.assert_allclose(row, f_row, rtol=1e-12)
    dX, dY = oracle.window_grad(X, Y, z, top["permX"], top["permY"], 1, 0, lse)
    fX, fY = oracle.full_ce_grad(X, Y, z, f_lse)
    assert rel_err(dX, fX) < 1e-12 and rel_err(dY, fY) < 1e-12


def test_window_loss_identical_rounds_equal_one_round():
    """r identical rounds compute every pair r times, each copy weighted by 1/r."""
    X, Y, z, B = _random_case(N=40, C=100, d=8, n_b=4, n_c=4, n_r=1)
    one = oracle.rece_forward(X, Y, z, B, 4, 1, 1)
    three_px = np.repeat(one["permX"], 3, 0)
    three_py = np.repeat(one["permY"], 3, 0)
    _, r1, l1 = oracle.window_loss(X, Y, z, one["permX"], one["permY"], 4, 1)
    _, r3, l3 = oracle.window_loss(X, Y, z, three_px, three_py, 4, 1)
    np.testing.assert_allclose(r3, r1, rtol=1e-12)
    g1 = oracle.window_grad(X, Y, z, one["permX"], one["permY"], 4, 1, l1)
    g3 = oracle.window_grad(X, Y, z, three_px, three_py, 4, 1, l3)
    assert rel_err(g3[0], g1[0]) < 1e-12 and rel_err(g3[1], g1[1]) < 1e-12


def test_window_grad_finite_differences_and_invariants():
    X, Y, z, B = _dyadic_case(N=6, C=20, d=3)
    top = oracle.rece_forward(X, Y, z, B, 3, 0, 1)
    px, py = top["permX"], top["permY"]
    _, _, lse = oracle.window_loss(X, Y, z, px, py, 3, 0)
    dloss = 0.9
    dX, dY = oracle.window_grad(X, Y, z, px, py, 3, 0, lse, dloss)
    h = 2.0 ** -10
    for name, A, G in (("X", X, dX), ("Y", Y, dY)):
        for idx in np.ndindex(A.shape):
            ls = []
            for sgn in (+1, -1):
                P = A.copy()
                P[idx] = P[idx] + np.float32(sgn * h)
                XX, YY = (P, Y) if name == "X" else (X, P)
                ls.append(oracle.window_loss(XX, YY, z, px, py, 3, 0)[0])
            fd = dloss * (ls[0] - ls[1]) / (2 * h)
            assert fd == pytest.approx(G[idx], abs=1e-6 * max(1.0, np.abs(G).max()))
    # every row's coefficients sum to zero -> the dY rows sum to the zero vector
    assert np.abs(dY.sum(0)).max() < 1e-12


def test_window_row_sample_matches_the_full_computation():
    X, Y, z, B = _random_case(N=50, C=140, d=8, n_b=3, n_c=5, n_r=2)
    top = oracle.rece_forward(X, Y, z, B, 5, 1, 1)
    px, py = top["permX"], top["permY"]
    _, row, lse = oracle.window_loss(X, Y, z, px, py, 5, 1)
    dX, _ = oracle.window_grad(X, Y, z, px, py, 5, 1, lse, 0.5)
    sample = np.array([3, 17, 49, 0, 22])
    _, srow, slse = oracle.window_loss(X, Y, z, px, py, 5, 1, rows=sample)
    np.testing.assert_array_equal(srow, row[sample])
    sX, _ = oracle.window_grad(X, Y, z, px, py, 5, 1, slse, 0.5, rows=sample)
    np.testing.assert_array_equal(sX, dX[sample])


# --------------------------------------------------------------------------- randn draw
def test_splitmix64_first_outputs_from_state_zero():
    """SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) started at state 0: its first three
    outputs as published with the generator (0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
    0x06C45D188009454F)."""
    assert oracle.splitmix64(0, 0) == 0xE220A8397B1DCDAF
    assert oracle.splitmix64(0, 1) == 0x6E789E6AA1B965F4
    assert oracle.splitmix64(0, 2) == 0x06C45D188009454F


def test_draw_projections_is_a_standard_normal_stream():
    """Algorithm 1's randn step as drawn by the oracle: against the normal law and the
    Box-Muller construction's own laws (Box and Muller 1958: for a pair (z0, z1),
    z0^2 + z1^2 is exponential with mean 2 and atan2(z1, z0) is uniform on (-pi, pi],
    independently), by Kolmogorov-Smirnov tests; independent pairs, calls and seeds."""
    from scipy import stats
    B = oracle.draw_projections(7, 3, 4, 1024, 256).ravel().astype(np.float64)
    n = B.size  # 2^20
    assert abs(B.mean()) < 5 / math.sqrt(n)
    assert abs(B.var() - 1.0) < 5 * math.sqrt(2.0 / n)
    assert stats.kstest(B, "norm").pvalue > 1e-3
    z0, z1 = B[0::2], B[1::2]
    assert stats.kstest(z0 ** 2 + z1 ** 2, "expon", args=(0, 2)).pvalue > 1e-3
    assert stats.kstest(np.arctan2(z1, z0), "uniform", args=(-math.pi, 2 * math.pi)).pvalue > 1e-3
    assert abs(np.corrcoef(z0, z1)[0, 1]) < 5 / math.sqrt(z0.size)
    # another call (step) and another seed: fresh, uncorrelated numbers
    B2 = oracle.draw_projections(7, 4, 4, 1024, 256).ravel().astype(np.float64)
    B3 = oracle.draw_projections(8, 3, 4, 1024, 256).ravel().astype(np.float64)
    assert abs(np.corrcoef(B, B2)[0, 1]) < 5 / math.sqrt(n)
    assert abs(np.corrcoef(B, B3)[0, 1]) < 5 / math.sqrt(n)
    # the same (seed, step) draws the same numbers; a shape is a prefix of the stream
    np.testing.assert_array_equal(oracle.draw_projections(7, 3, 4, 1024, 256).ravel(), B)
    np.testing.assert_array_equal(oracle.draw_projections(7, 3, 1, 1, 99).ravel(), B[:99])
