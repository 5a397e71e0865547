"""Shared helpers of the GPU tests: run the CUDA path through the C ABI and the oracle
on the same seeded inputs, and compare."""
import numpy as np
import torch

import oracle
from reduced_cross_entropy_b200 import ops, synth


def to_dev(a: np.ndarray, dtype: str):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def max_rel(a, b):
    """max |a - b| / max |b| over all elements (max-norm relative error)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.max(np.abs(b)) if b.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(a))) if a.size else 0.0
    return float(np.max(np.abs(a - b)) / den)


def run_gpu(w: synth.Workload, X, Y, t, B, flags=0, dloss=1.0, use_logits=True,
            auto_buckets=False):
    """Whole path on the GPU.  Returns a dict of numpy arrays.  auto_buckets: the plan is
    created with n_b = n_c = 0 (the library picks the pages' n_b*), which must resolve to
    w's n_b and n_c."""
    plan = ops.Plan(w.N, w.C, w.d, 0 if auto_buckets else w.n_b, 0 if auto_buckets else w.n_c,
                    w.n_ec, w.n_r, w.k, mode=w.dtype, flags=flags)
    assert (plan.n_b, plan.n_c) == (w.n_b, w.n_c)
    Xd, Yd, Bd = to_dev(X, w.dtype), to_dev(Y, w.dtype), to_dev(B, w.dtype)
    td = torch.from_numpy(t).cuda()
    ws = plan.workspace()
    ops.bucketize_sort(plan, Bd, Xd, Yd, ws)
    bx, by = (a.cpu().numpy() for a in plan.bucket_ids(ws))
    px, py = (a.cpu().numpy() for a in plan.permutations(ws))
    loss, row, sel, lse, logits = ops.loss_fwd(plan, Xd, Yd, td, ws)
    dl = torch.tensor([dloss], dtype=torch.float32, device="cuda")
    dX, dY = ops.loss_bwd(plan, Xd, Yd, td, sel, lse, dl, ws,
                          logits=logits if use_logits else None)
    status = ops.device_status(ws)
    # status area: flags, inexact rows, overflowed lists, rows the merge spilled, items
    # the sampled selection handed to the exact kernel
    words = ws[:32].view(torch.int32).cpu().numpy()
    return dict(bx=bx, by=by, permX=px, permY=py, loss=float(loss.item()), words=words,
                row_loss=row.cpu().numpy(), selected=sel.cpu().numpy(), lse=lse.cpu().numpy(),
                dX=dX.cpu().numpy(), dY=dY.cpu().numpy(), status=status, plan=plan,
                logits=logits.cpu().numpy())


def run_oracle(w: synth.Workload, X, Y, t, B, dloss=1.0):
    out = oracle.rece_forward(X, Y, t, B, w.n_c, w.n_ec, w.k)
    dX, dY = oracle.rece_grad(X, Y, t, out["selected"], out["lse"], dloss)
    out.update(dX=dX, dY=dY)
    return out
