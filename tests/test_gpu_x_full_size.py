"""Parity at the full sizes of the benchmark workloads, in the launch configuration the
benchmark times (its seed-0 inputs, default flags, the logits handed to the backward).

The GPU runs the whole path once through the C ABI.  The oracle then checks, one by one,
what it can afford at these sizes -- sampled rows (bucket ids, selected sets, row losses,
dX rows) and sampled items (bucket ids, dY rows: the most frequent positive, the most
selected negative, the first and last items, random ones, one nobody touches) -- and
properties that hold at any size are checked on whole arrays (the orders are the stable
argsort of the bucket ids; every selection is distinct, free of the positive and inside
the row's windows).  Floating point decides the bucket ids and the selection, so the
GPU's own orders feed the later checks and a differing bucket must be a near-tie."""
import bisect

import numpy as np
import pytest
import torch

import oracle
from gpu_common import max_rel, to_dev
from reduced_cross_entropy_b200 import _lib, ops, synth

pytestmark = pytest.mark.gpu

ROWS = 24    # sampled rows
RANDOM_ITEMS = 4


def _windows(M_side, K_side, n_c, n_ec):
    """Chunk starts of both sides: a sorted row p of chunk c sees the sorted catalogue
    positions [start(c - n_ec), start(c + n_ec + 1)) (clipped)."""
    rs = [oracle.chunk_start(c, M_side, n_c) for c in range(n_c + 1)]
    ks = [oracle.chunk_start(c, K_side, n_c) for c in range(n_c + 1)]

    def window(p):
        c = bisect.bisect_right(rs, p) - 1
        return ks[max(c - n_ec, 0)], ks[min(c + n_ec + 1, n_c)]
    return window


@pytest.mark.parametrize("name", ["sasrec", "large", "very_large", "lm"])
def test_full_size_sampled_parity(name):
    w = synth.WORKLOADS[name]
    X, Y, t = synth.make_inputs(w, seed=0)
    B = synth.projections(0, 0, w.n_r, w.n_b, w.d, w.dtype)
    plan = ops.Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype)
    Xd, Yd, Bd = to_dev(X, w.dtype), to_dev(Y, w.dtype), to_dev(B, w.dtype)
    td = torch.from_numpy(t).cuda()
    ws = plan.workspace()
    ops.bucketize_sort(plan, Bd, Xd, Yd, ws)
    bx, by = (a.cpu().numpy() for a in plan.bucket_ids(ws))
    px, py = (a.cpu().numpy() for a in plan.permutations(ws))
    _, row, sel_d, lse_d, logits = ops.loss_fwd(plan, Xd, Yd, td, ws)
    dX, dY = ops.loss_bwd(plan, Xd, Yd, td, sel_d, lse_d, torch.ones(1, device="cuda"), ws,
                          logits=logits)
    assert ops.device_status(ws) & ~_lib.DEVICE_INEXACT == 0
    sel = sel_d.cpu().numpy()
    row = row.cpu().numpy()

    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, ROWS - 2, replace=False)]))
    counts = np.bincount(sel[sel >= 0], minlength=w.C)
    touched = counts + np.bincount(t, minlength=w.C)
    untouched = np.nonzero(touched == 0)[0]
    items = [int(np.bincount(t, minlength=w.C).argmax()), int(counts.argmax()), 0, w.C - 1]
    items += rng.choice(np.nonzero(touched)[0], RANDOM_ITEMS, replace=False).tolist()
    items = sorted(set(items))
    if len(untouched):
        items.append(int(untouched[len(untouched) // 2]))

    # step 1: bucket ids of a sample of rows and items (8192 of each, the checked rows and
    # items among them) against the oracle's argmax: a differing id must be a near-tie,
    # and at most 1e-3 of them may differ
    many_rows = np.union1d(rows, rng.choice(w.N, min(w.N, 8192), replace=False))
    many_items = np.union1d(items, rng.choice(w.C, min(w.C, 8192), replace=False))
    for r in range(w.n_r):
        for V, ids, got in ((X, many_rows, bx[r]), (Y, many_items, by[r])):
            want = oracle.bucketize(V[ids], B[r])
            diff = np.nonzero(got[ids] != want)[0]
            assert len(diff) <= 1e-3 * len(ids), (len(diff), len(ids))
            P = V[ids[diff]].astype(np.float64) @ B[r].astype(np.float64).T
            for a, j in enumerate(diff):
                assert abs(P[a, got[ids[j]]] - P[a, want[j]]) <= 1e-5 * np.abs(P[a]).max()
    # step 2: the orders are the stable argsort of the GPU's bucket ids (whole arrays)
    for r in range(w.n_r):
        np.testing.assert_array_equal(px[r], oracle.stable_argsort(bx[r]))
        np.testing.assert_array_equal(py[r], oracle.stable_argsort(by[r]))

    # steps 3-4: the sampled rows' selections, on the GPU's orders
    osel, _, _ = oracle.select(X, Y, t, px, py, w.n_c, w.n_ec, w.k, rows=rows)
    hit = tot = 0
    inv_x = np.empty_like(px)
    inv_y = np.empty_like(py)
    for r in range(w.n_r):
        inv_x[r][px[r]] = np.arange(w.N, dtype=np.int32)
        inv_y[r][py[r]] = np.arange(w.C, dtype=np.int32)
    window = _windows(w.N, w.C, w.n_c, w.n_ec)
    for a, i in enumerate(rows):
        g, o = sel[i][sel[i] >= 0], osel[a][osel[a] >= 0]
        hit += len(set(g.tolist()) & set(o.tolist()))
        tot += len(o)
        assert len(set(g.tolist())) == len(g) and int(t[i]) not in set(g.tolist())
        inside = np.zeros(len(g), bool)
        for r in range(w.n_r):
            w0, w1 = window(int(inv_x[r][i]))
            q = inv_y[r][g]
            inside |= (q >= w0) & (q < w1)
        assert inside.all()
    assert hit >= 0.99 * tot, (hit, tot)

    # step 5: the sampled rows' losses, for the GPU's selection
    _, o_row, o_lse = oracle.rece_loss(X[rows], Y, t[rows], sel[rows])
    assert max_rel(row[rows], o_row) <= 1e-4

    # step 6: dX rows of the sampled rows, dY rows of the sampled items
    oX = oracle.rece_grad_rows(X, Y, t, rows, sel[rows], o_lse)
    assert max_rel(dX[torch.from_numpy(rows).cuda()].cpu().numpy(), oX) <= 1e-3
    holders = np.nonzero(np.isin(sel, items).any(axis=1) | np.isin(t, items))[0]
    _, _, h_lse = oracle.rece_loss(X[holders], Y, t[holders], sel[holders])
    oY = oracle.rece_grad_items(X, Y, t, holders, sel[holders], h_lse, items)
    gY = dY[torch.tensor(items, device="cuda")].cpu().numpy()
    assert max_rel(gY, oY) <= 1e-3
    if len(untouched):
        assert np.all(gY[-1] == 0.0)  # an item nobody touches gets exactly zero
