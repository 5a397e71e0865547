"""Parity of the sampled baselines (RECE section 2, equations (1) BCE+ and (2) CE-) on
the GPU against the oracle, through the C ABI: losses, logits, lse and gradients,
element by element, on seeded inputs that span several warps' rows, ragged sizes,
padding, repeated samples and the positive drawn as a negative."""
import numpy as np
import pytest
import torch

import oracle
from reduced_cross_entropy_b200 import ops, synth

from gpu_common import max_rel, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-4  # fp32 arithmetic against the fp64 oracle on the same (bf16-rounded) inputs

KINDS = {"ce_minus": oracle.SAMPLED_CE_MINUS, "bce_plus": oracle.SAMPLED_BCE_PLUS}


def _case(N, C, d, n, dtype, seed, alpha=1.0):
    w = synth.Workload("sampled", N=N, C=C, d=d, dtype=dtype, n_b=1, n_c=1, n_ec=0, n_r=1,
                       k=1, target_alpha=alpha)
    X, Y, t = synth.make_inputs(w, seed=seed)
    neg = synth.uniform_negatives(seed, N, C, n)
    if N > 2 and n > 2:
        neg[0, :] = t[0]            # the positive drawn as every negative
        neg[1, 1] = neg[1, 0]       # a repeated sample
        neg[2, -2:] = -1            # padding
    return X, Y, t, neg


def _run(kind, X, Y, t, neg, dtype, dloss=1.0, use_logits=True):
    Xd, Yd = to_dev(X, dtype), to_dev(Y, dtype)
    td, nd = torch.from_numpy(t).cuda(), torch.from_numpy(neg).cuda()
    loss, row, logits, lse, ws = ops.sampled_fwd(kind, Xd, Yd, td, nd)
    dl = torch.tensor([dloss], dtype=torch.float32, device="cuda")
    dX, dY = ops.sampled_bwd(kind, Xd, Yd, td, nd, lse, dl, ws,
                             logits=logits if use_logits else None)
    return dict(loss=loss.item(), row=row.cpu().numpy(), logits=logits.cpu().numpy(),
                lse=lse.cpu().numpy(), dX=dX.cpu().numpy(), dY=dY.cpu().numpy(),
                status=ops.device_status(ws))


@pytest.mark.parametrize("kind", list(KINDS))
@pytest.mark.parametrize("dtype,N,C,d,n", [
    ("fp32", 1003, 5000, 64, 100),     # ragged row count, d % 8 == 0 kernels
    ("fp32", 517, 777, 40, 33),        # d % 8 != 0 kernels, ragged slots
    ("bf16", 1003, 5000, 64, 100),
    ("bf16", 300, 20000, 256, 255),
])
def test_sampled_parity(kind, dtype, N, C, d, n):
    X, Y, t, neg = _case(N, C, d, n, dtype, seed=N + n)
    g = _run(kind, X, Y, t, neg, dtype, dloss=1.5)
    o_loss, o_row, o_lse = oracle.sampled_loss(KINDS[kind], X, Y, t, neg)
    assert g["status"] == 0
    assert abs(g["loss"] - o_loss) <= TOL * abs(o_loss)
    assert max_rel(g["row"], o_row) <= TOL
    if kind == "ce_minus":
        assert max_rel(g["lse"], o_lse) <= TOL
    # logits: slot 0 the positive, slot s the negative s-1 (padding 0)
    Xo, Yo = X.astype(np.float64), Y.astype(np.float64)
    ids = np.concatenate([t[:, None], neg], 1)
    ref = np.einsum("id,ind->in", Xo, Yo[np.maximum(ids, 0)])
    ref[ids < 0] = 0.0
    assert max_rel(g["logits"], ref) <= TOL
    fX, fY = oracle.sampled_grad(KINDS[kind], X, Y, t, neg, o_lse, 1.5)
    assert max_rel(g["dX"], fX) <= TOL
    assert max_rel(g["dY"], fY) <= TOL


@pytest.mark.parametrize("kind", list(KINDS))
def test_sampled_recomputed_logits_and_determinism(kind):
    X, Y, t, neg = _case(700, 3000, 64, 64, "bf16", seed=3)
    a = _run(kind, X, Y, t, neg, "bf16", use_logits=False)
    b = _run(kind, X, Y, t, neg, "bf16", use_logits=False)
    c = _run(kind, X, Y, t, neg, "bf16", use_logits=True)
    for key in ("row", "logits", "dX", "dY"):
        assert np.array_equal(a[key], b[key]), key     # bit for bit, run to run
    _, _, o_lse = oracle.sampled_loss(KINDS[kind], X, Y, t, neg)
    fX, fY = oracle.sampled_grad(KINDS[kind], X, Y, t, neg, o_lse)
    assert max_rel(a["dX"], fX) <= TOL and max_rel(a["dY"], fY) <= TOL
    assert max_rel(c["dY"], fY) <= TOL


def test_ce_minus_over_every_other_item_is_full_ce():
    """All C - 1 other items sampled once: CE- is the full cross-entropy (eq. 3)."""
    N, C, d = 200, 300, 32
    X, Y, t, _ = _case(N, C, d, 0, "fp32", seed=9)
    neg = np.array([[j for j in range(C) if j != t[i]] for i in range(N)], np.int32)
    g = _run("ce_minus", X, Y, t, neg, "fp32")
    f_loss, f_row, f_lse = oracle.full_ce_loss(X, Y, t)
    assert abs(g["loss"] - f_loss) <= TOL * f_loss
    fX, fY = oracle.full_ce_grad(X, Y, t, f_lse)
    assert max_rel(g["dX"], fX) <= TOL and max_rel(g["dY"], fY) <= TOL


@pytest.mark.parametrize("kind", list(KINDS))
def test_sampled_edge_cases(kind):
    # no negatives: CE- is exactly 0, BCE+ is softplus(-l+)
    X, Y, t, _ = _case(65, 90, 16, 0, "fp32", seed=1)
    neg = np.zeros((65, 0), np.int32)
    g = _run(kind, X, Y, t, neg, "fp32")
    o_loss, o_row, o_lse = oracle.sampled_loss(KINDS[kind], X, Y, t, neg)
    assert max_rel(g["row"], o_row) <= TOL
    if kind == "ce_minus":
        assert np.all(g["row"] == 0.0)
    fX, fY = oracle.sampled_grad(KINDS[kind], X, Y, t, neg, o_lse)
    assert max_rel(g["dX"], fX) <= TOL and max_rel(g["dY"], fY) <= TOL
    # all-padding rows and an empty batch
    X, Y, t, neg = _case(40, 50, 8, 6, "fp32", seed=2)
    neg[:] = -1
    g = _run(kind, X, Y, t, neg, "fp32")
    assert max_rel(g["row"], oracle.sampled_loss(KINDS[kind], X, Y, t, neg)[1]) <= TOL
    Xe = np.zeros((0, 8), np.float32)
    g = _run(kind, Xe, Y, np.zeros(0, np.int32), np.zeros((0, 6), np.int32), "fp32")
    assert g["loss"] == 0.0 and np.all(g["dY"] == 0.0)


def test_sampled_bad_ids_raise_the_device_flag():
    X, Y, t, neg = _case(64, 100, 8, 4, "fp32", seed=4)
    neg[5, 2] = 100                 # == C
    g = _run("bce_plus", X, Y, t, neg, "fp32")
    assert g["status"] & 0x1
