"""PyTorch binding of the C ABI: argument checks and pointer marshalling only.

Every step of the loss runs in the CUDA library; torch supplies device memory, the
current stream and autograd plumbing.  Output buffers are allocated here with torch
(the library itself never allocates).
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib

_MODES = {"fp32": _lib.MODE_FP32_EXACT, "bf16": _lib.MODE_BF16}
_DTYPES = {_lib.MODE_FP32_EXACT: torch.float32, _lib.MODE_BF16: torch.bfloat16}


def _vp(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class Plan:
    """Host-side plan (validated config + workspace layout) of one problem size."""

    def __init__(self, N: int, C: int, d: int, n_b: int, n_c: int, n_ec: int = 1,
                 n_r: int = 1, k: int = 256, mode: str = "bf16", flags: int = 0):
        self.mode = _MODES[mode] if isinstance(mode, str) else int(mode)
        self.cfg = _lib.Config(N, C, d, n_b, n_c, n_ec, n_r, k, self.mode, flags)
        h = ctypes.c_void_p()
        L = _lib.lib()
        _lib.check(L.rece_plan_create(ctypes.byref(self.cfg), ctypes.byref(h)),
                   "rece_plan_create")
        self._h = h
        # the configuration as the library resolved it (n_b = n_c = 0: the pages' n_b*)
        _lib.check(L.rece_plan_get_config(h, ctypes.byref(self.cfg)), "rece_plan_get_config")
        size = ctypes.c_size_t()
        _lib.check(L.rece_plan_workspace_size(h, ctypes.byref(size)), "workspace_size")
        self.workspace_bytes = int(size.value)
        self.layout = _lib.WorkspaceLayout()
        _lib.check(L.rece_plan_workspace_layout(h, ctypes.byref(self.layout)), "layout")

    def __del__(self):
        h = getattr(self, "_h", None)
        lib = getattr(_lib, "_lib", None) if _lib is not None else None  # None at exit
        if h is not None and h.value and lib is not None:
            lib.rece_plan_destroy(h)
            self._h = None

    @property
    def dtype(self):
        return _DTYPES[self.mode]

    @property
    def paths(self) -> int:
        """OR of _lib.PATH_* flags: which kernels this plan runs."""
        v = ctypes.c_uint32()
        _lib.check(_lib.lib().rece_plan_paths(self._h, ctypes.byref(v)), "rece_plan_paths")
        return int(v.value)

    def __getattr__(self, name):
        if name in ("N", "C", "d", "n_b", "n_c", "n_ec", "n_r", "k", "flags"):
            return getattr(self.cfg, name)
        raise AttributeError(name)

    def workspace(self, device="cuda") -> torch.Tensor:
        return torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8, device=device)

    # views of the intermediates held in the workspace (valid after bucketize_sort)
    def _ws_view(self, ws, offset, n):
        return ws[offset:offset + 4 * n].view(torch.int32)

    def bucket_ids(self, ws):
        c = self.cfg
        return (self._ws_view(ws, self.layout.bucket_x, c.n_r * c.N).view(c.n_r, c.N),
                self._ws_view(ws, self.layout.bucket_y, c.n_r * c.C).view(c.n_r, c.C))

    def permutations(self, ws):
        c = self.cfg
        return (self._ws_view(ws, self.layout.perm_x, c.n_r * c.N).view(c.n_r, c.N),
                self._ws_view(ws, self.layout.perm_y, c.n_r * c.C).view(c.n_r, c.C))

    def bucket_starts_y(self, ws):
        s = self.layout.bucket_start_stride
        return self._ws_view(ws, self.layout.bucket_start_y, self.cfg.n_r * s).view(
            self.cfg.n_r, s)


def _check_ws(plan: Plan, ws: torch.Tensor):
    if ws.device.type != "cuda" or ws.dtype != torch.uint8 or ws.numel() < plan.workspace_bytes:
        raise ValueError("workspace must be a CUDA uint8 tensor of plan.workspace_bytes bytes")


def draw_projections(plan: Plan, seed: int, step: int, out=None, stream=None):
    """Algorithm 1's random vectors B [n_r, n_b, d] of call `step` of a run seeded with
    `seed`, drawn on the device (rece_draw_projections).  Returns `out` (allocated when
    None) in the plan's element type."""
    c = plan.cfg
    if out is None:
        out = torch.empty((c.n_r, c.n_b, c.d), dtype=plan.dtype, device="cuda")
    _need(out, "B", plan.dtype, (c.n_r, c.n_b, c.d))
    _lib.check(_lib.lib().rece_draw_projections(plan._h, seed & (2**64 - 1), step & (2**64 - 1),
                                                _vp(out), _stream(stream)),
               "rece_draw_projections")
    return out


def bucketize_sort(plan: Plan, B, X, Y, ws, stream=None):
    """Steps 1-2: bucket ids and stable per-round orders (into the workspace)."""
    c = plan.cfg
    _need(B, "B", plan.dtype, (c.n_r, c.n_b, c.d))
    _need(X, "X", plan.dtype, (c.N, c.d))
    _need(Y, "Y", plan.dtype, (c.C, c.d))
    _check_ws(plan, ws)
    _lib.check(_lib.lib().rece_bucketize_sort(plan._h, _vp(B), _vp(X), _vp(Y), _vp(ws),
                                              ws.numel(), _stream(stream)),
               "rece_bucketize_sort")


def loss_fwd(plan: Plan, X, Y, targets, ws, *, want_row_loss: bool = True,
             want_logits: bool = True, stream=None):
    """Steps 3-5.  Returns (loss [1], row_loss [N] or None, selected [N,k], lse [N],
    logits [N,k+1] or None)."""
    c = plan.cfg
    _need(X, "X", plan.dtype, (c.N, c.d))
    _need(Y, "Y", plan.dtype, (c.C, c.d))
    _need(targets, "targets", torch.int32, (c.N,))
    _check_ws(plan, ws)
    dev = X.device
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    row = torch.empty(c.N, dtype=torch.float32, device=dev) if want_row_loss else None
    sel = torch.empty(c.N, c.k, dtype=torch.int32, device=dev)
    lse = torch.empty(c.N, dtype=torch.float32, device=dev)
    logits = torch.empty(c.N, c.k + 1, dtype=torch.float32, device=dev) if want_logits else None
    _lib.check(_lib.lib().rece_loss_fwd(plan._h, _vp(X), _vp(Y), _vp(targets), _vp(ws),
                                        ws.numel(), _vp(loss), _vp(row), _vp(sel), _vp(lse),
                                        _vp(logits), _stream(stream)), "rece_loss_fwd")
    return loss, row, sel, lse, logits


def loss_bwd(plan: Plan, X, Y, targets, selected, lse, dloss, ws, logits=None, stream=None):
    """Step 6.  Returns (dX [N,d] fp32, dY [C,d] fp32).  `logits` from loss_fwd spares
    recomputing the selected logits (None: recompute them)."""
    c = plan.cfg
    _need(X, "X", plan.dtype, (c.N, c.d))
    _need(Y, "Y", plan.dtype, (c.C, c.d))
    _need(targets, "targets", torch.int32, (c.N,))
    _need(selected, "selected", torch.int32, (c.N, c.k))
    _need(lse, "lse", torch.float32, (c.N,))
    _need(dloss, "dloss", torch.float32, (1,))
    if logits is not None:
        _need(logits, "logits", torch.float32, (c.N, c.k + 1))
    _check_ws(plan, ws)
    dX = torch.empty(c.N, c.d, dtype=torch.float32, device=X.device)
    dY = torch.empty(c.C, c.d, dtype=torch.float32, device=X.device)
    _lib.check(_lib.lib().rece_loss_bwd(plan._h, _vp(X), _vp(Y), _vp(targets), _vp(selected),
                                        _vp(lse), _vp(logits), _vp(dloss), _vp(ws), ws.numel(),
                                        _vp(dX), _vp(dY), _stream(stream)), "rece_loss_bwd")
    return dX, dY


def device_status(ws, stream=None) -> int:
    """Synchronise and read the workspace status word (RECE_DEVICE_* bits)."""
    flags = ctypes.c_uint32(0)
    st = _lib.lib().rece_get_device_status(_vp(ws), ctypes.byref(flags), _stream(stream))
    if st not in (_lib.RECE_OK, 5, 6):
        _lib.check(st, "rece_get_device_status")
    return int(flags.value)


def full_ce_workspace_bytes(N, C, d, mode="bf16") -> int:
    size = ctypes.c_size_t()
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    _lib.check(_lib.lib().rece_full_ce_workspace_size(N, C, d, m, ctypes.byref(size)),
               "rece_full_ce_workspace_size")
    return int(size.value)


def full_ce_fwd(X, Y, targets, ws=None, stream=None):
    """Exact fused full CE forward.  Returns (loss [1], row_loss [N], lse [N], ws)."""
    N, d = X.shape
    C = Y.shape[0]
    mode = _lib.MODE_BF16 if X.dtype == torch.bfloat16 else _lib.MODE_FP32_EXACT
    _need(X, "X", _DTYPES[mode], (N, d))
    _need(Y, "Y", _DTYPES[mode], (C, d))
    _need(targets, "targets", torch.int32, (N,))
    nbytes = full_ce_workspace_bytes(N, C, d, mode)
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=X.device)
    loss = torch.empty(1, dtype=torch.float32, device=X.device)
    row = torch.empty(N, dtype=torch.float32, device=X.device)
    lse = torch.empty(N, dtype=torch.float32, device=X.device)
    _lib.check(_lib.lib().rece_full_ce_fwd(N, C, d, mode, _vp(X), _vp(Y), _vp(targets),
                                           _vp(ws), ws.numel(), _vp(loss), _vp(row), _vp(lse),
                                           _stream(stream)), "rece_full_ce_fwd")
    return loss, row, lse, ws


def full_ce_bwd(X, Y, targets, lse, dloss, ws, stream=None):
    N, d = X.shape
    C = Y.shape[0]
    mode = _lib.MODE_BF16 if X.dtype == torch.bfloat16 else _lib.MODE_FP32_EXACT
    _need(lse, "lse", torch.float32, (N,))
    _need(dloss, "dloss", torch.float32, (1,))
    dX = torch.empty(N, d, dtype=torch.float32, device=X.device)
    dY = torch.empty(C, d, dtype=torch.float32, device=X.device)
    _lib.check(_lib.lib().rece_full_ce_bwd(N, C, d, mode, _vp(X), _vp(Y), _vp(targets),
                                           _vp(lse), _vp(dloss), _vp(ws), ws.numel(), _vp(dX),
                                           _vp(dY), _stream(stream)), "rece_full_ce_bwd")
    return dX, dY


def optimal_buckets(N: int, C: int, n_ec: int, alpha_bc: float):
    """(n_b*, n_c*) of the least memory (RECE section 3), for alpha_bc = n_b / n_c."""
    nb, nc = ctypes.c_int32(), ctypes.c_int32()
    _lib.check(_lib.lib().rece_optimal_buckets(N, C, n_ec, float(alpha_bc), ctypes.byref(nb),
                                               ctypes.byref(nc)), "rece_optimal_buckets")
    return int(nb.value), int(nc.value)


def memory_model_elements(N: int, C: int, n_ec: int, n_r: int, alpha_bc: float) -> float:
    """The pages' memory model of the method at n_b*, in logit elements."""
    v = ctypes.c_double()
    _lib.check(_lib.lib().rece_memory_model_elements(N, C, n_ec, n_r, float(alpha_bc),
                                                     ctypes.byref(v)),
               "rece_memory_model_elements")
    return float(v.value)


_KINDS = {"ce_minus": _lib.SAMPLED_CE_MINUS, "bce_plus": _lib.SAMPLED_BCE_PLUS}


def _kind(kind) -> int:
    return _KINDS[kind] if isinstance(kind, str) else int(kind)


def sampled_workspace_bytes(kind, N, C, d, n, mode="bf16") -> int:
    size = ctypes.c_size_t()
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    _lib.check(_lib.lib().rece_sampled_workspace_size(_kind(kind), N, C, d, n, m,
                                                      ctypes.byref(size)),
               "rece_sampled_workspace_size")
    return int(size.value)


def sampled_fwd(kind, X, Y, targets, negatives, ws=None, stream=None):
    """Sampled baseline forward: kind "ce_minus" (RECE section 2, eq. 2) or "bce_plus"
    (eq. 1) over negatives [N, n] int32 (ids < 0: padding).
    Returns (loss [1], row_loss [N], logits [N, n+1], lse [N], ws)."""
    N, d = X.shape
    C = Y.shape[0]
    n = negatives.shape[1]
    mode = _lib.MODE_BF16 if X.dtype == torch.bfloat16 else _lib.MODE_FP32_EXACT
    _need(X, "X", _DTYPES[mode], (N, d))
    _need(Y, "Y", _DTYPES[mode], (C, d))
    _need(targets, "targets", torch.int32, (N,))
    _need(negatives, "negatives", torch.int32, (N, n))
    nbytes = sampled_workspace_bytes(kind, N, C, d, n, mode)
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=X.device)
    loss = torch.empty(1, dtype=torch.float32, device=X.device)
    row = torch.empty(N, dtype=torch.float32, device=X.device)
    logits = torch.empty(N, n + 1, dtype=torch.float32, device=X.device)
    lse = torch.empty(N, dtype=torch.float32, device=X.device)
    _lib.check(_lib.lib().rece_sampled_fwd(_kind(kind), N, C, d, n, mode, _vp(X), _vp(Y),
                                           _vp(targets), _vp(negatives), _vp(ws), ws.numel(),
                                           _vp(loss), _vp(row), _vp(logits), _vp(lse),
                                           _stream(stream)), "rece_sampled_fwd")
    return loss, row, logits, lse, ws


def sampled_bwd(kind, X, Y, targets, negatives, lse, dloss, ws, logits=None, stream=None):
    """Gradients of the sampled baseline (negatives held constant): (dX, dY) fp32."""
    N, d = X.shape
    C = Y.shape[0]
    n = negatives.shape[1]
    mode = _lib.MODE_BF16 if X.dtype == torch.bfloat16 else _lib.MODE_FP32_EXACT
    _need(lse, "lse", torch.float32, (N,))
    _need(dloss, "dloss", torch.float32, (1,))
    if logits is not None:
        _need(logits, "logits", torch.float32, (N, n + 1))
    dX = torch.empty(N, d, dtype=torch.float32, device=X.device)
    dY = torch.empty(C, d, dtype=torch.float32, device=X.device)
    _lib.check(_lib.lib().rece_sampled_bwd(_kind(kind), N, C, d, n, mode, _vp(X), _vp(Y),
                                           _vp(targets), _vp(negatives), _vp(logits), _vp(lse),
                                           _vp(dloss), _vp(ws), ws.numel(), _vp(dX), _vp(dY),
                                           _stream(stream)), "rece_sampled_bwd")
    return dX, dY


class _ReceLossFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, Y, targets, B, plan, ws):
        bucketize_sort(plan, B, X, Y, ws)
        loss, _, sel, lse, logits = loss_fwd(plan, X, Y, targets, ws, want_row_loss=False)
        ctx.save_for_backward(X, Y, targets, sel, lse, logits)
        ctx.plan, ctx.ws = plan, ws
        return loss.reshape(())

    @staticmethod
    def backward(ctx, grad):
        X, Y, targets, sel, lse, logits = ctx.saved_tensors
        dloss = grad.detach().float().reshape(1).contiguous()
        dX, dY = loss_bwd(ctx.plan, X, Y, targets, sel, lse, dloss, ctx.ws, logits=logits)
        return dX.to(X.dtype), dY.to(Y.dtype), None, None, None, None


def rece_loss(X, Y, targets, B, plan: Plan, ws=None):
    """Reduced cross-entropy loss with autograd (gradients for X and Y).

    B: the random vectors of this call [n_r, n_b, d] (afresh every step), or a pair
    (seed, step), for which the library draws them on the device (draw_projections)."""
    if ws is None:
        ws = plan.workspace(X.device)
    if isinstance(B, tuple):
        B = draw_projections(plan, int(B[0]), int(B[1]))
    return _ReceLossFn.apply(X, Y, targets, B, plan, ws)
