"""CPU oracle of the reduced cross-entropy (RECE / SCE) loss -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA library and never calls it.

Every function takes fp32 numpy arrays (bf16 inputs are passed as their exact fp32
upcast) and follows the definitions cited in ``rece_oracle.c``:

* ``bucketize``     -- RECE paper, section 3, Algorithm 1 (argmax over random vectors)
* ``stable_argsort``-- Algorithm 1's argsort, read as a stable sort
* ``chunk_start``   -- Algorithm 1's chunk sets, start of chunk c = ceil(c*M/n_c)
* ``select``        -- candidates of the chunk windows over all rounds, positive removed,
                       de-duplicated, the k best by (score desc, item asc) (SCE abstract)
* ``rece_loss`` / ``rece_grad``       -- Algorithm 1's loss, equation (4) on the subset
* ``rece_grad_rows`` / ``rece_grad_items`` -- rece_grad's dX rows / dY rows for a sample of
                       row or item ids only (the same sums, restricted; numpy fp64)
* ``full_ce_loss`` / ``full_ce_grad`` -- equations (3) and (4) over the whole catalogue
* ``window_loss`` / ``window_grad`` -- Algorithm 1 as printed: every window item a
                       negative, duplicates across rounds corrected by ln(count)
* ``optimal_buckets`` / ``memory_model_elements`` -- section 3's n_b* and memory model
* ``sampled_loss`` / ``sampled_grad`` -- the sampled baselines of section 2: CE- (eq. 2,
                       kind 0) and BCE+ (eq. 1, kind 1) over given negatives
* ``rece_forward``  -- the whole forward path, steps 1 to 5, given the random vectors B
* ``draw_projections`` / ``splitmix64`` -- Algorithm 1's randn step as a counter-based
                       stream of (seed, step): SplitMix64 outputs, Box-Muller normals
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.oracle_bucketize.argtypes = [f32p, i64, i32, f32p, i32, i32p]
        lib.oracle_bucketize.restype = None
        lib.oracle_stable_argsort.argtypes = [i32p, i64, i32p]
        lib.oracle_stable_argsort.restype = None
        lib.oracle_chunk_start.argtypes = [i64, i64, i64]
        lib.oracle_chunk_start.restype = i64
        u64 = ctypes.c_uint64
        lib.oracle_splitmix64.argtypes = [u64, u64]
        lib.oracle_splitmix64.restype = u64
        lib.oracle_draw_projections.argtypes = [u64, u64, i64, f32p]
        lib.oracle_draw_projections.restype = None
        i64p_or_null = ctypes.c_void_p
        lib.oracle_select.argtypes = [f32p, f32p, i32p, i64, i64, i32, i32, i32, i32, i32,
                                      i32p, i32p, i64p_or_null, i64, i32p, f32p, i64p]
        lib.oracle_select.restype = None
        lib.oracle_rece_loss.argtypes = [f32p, f32p, i32p, i64, i32, i32, i32p, f64p, f64p,
                                         f64p]
        lib.oracle_rece_loss.restype = None
        lib.oracle_rece_grad.argtypes = [f32p, f32p, i32p, i64, i64, i32, i32, i32p, f64p,
                                         ctypes.c_double, f64p, f64p]
        lib.oracle_rece_grad.restype = None
        lib.oracle_full_ce_loss.argtypes = [f32p, f32p, i32p, i64, i64, i32, f64p, f64p, f64p]
        lib.oracle_full_ce_loss.restype = None
        lib.oracle_full_ce_grad.argtypes = [f32p, f32p, i32p, i64, i64, i32, f64p,
                                            ctypes.c_double, f64p, f64p]
        lib.oracle_full_ce_grad.restype = None
        lib.oracle_sampled_loss.argtypes = [i32, f32p, f32p, i32p, i64, i32, i32, i32p, f64p,
                                            f64p, f64p]
        lib.oracle_sampled_loss.restype = None
        lib.oracle_sampled_grad.argtypes = [i32, f32p, f32p, i32p, i64, i64, i32, i32, i32p,
                                            f64p, ctypes.c_double, f64p, f64p]
        lib.oracle_sampled_grad.restype = None
        lib.oracle_window_loss.argtypes = [f32p, f32p, i32p, i64, i64, i32, i32, i32, i32,
                                           i32p, i32p, i64p_or_null, i64, f64p, f64p, f64p]
        lib.oracle_window_loss.restype = None
        lib.oracle_window_grad.argtypes = [f32p, f32p, i32p, i64, i64, i32, i32, i32, i32,
                                           i32p, i32p, i64p_or_null, i64, f64p,
                                           ctypes.c_double, f64p, f64p]
        lib.oracle_window_grad.restype = None
        lib.oracle_dot_f32.argtypes = [f32p, f32p, i32]
        lib.oracle_dot_f32.restype = ctypes.c_float
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def dot_f32(a, b) -> np.float32:
    """fp32 fmaf-chain inner product, the score every integer decision is taken on."""
    a, b = _f32(a), _f32(b)
    return np.float32(_load().oracle_dot_f32(a, b, a.shape[0]))


def bucketize(V, B) -> np.ndarray:
    """Bucket id of every row of V: argmax_b <B[b], v> (ties to the lowest b)."""
    V, B = _f32(V), _f32(B)
    out = np.empty(V.shape[0], np.int32)
    _load().oracle_bucketize(V, V.shape[0], V.shape[1], B, B.shape[0], out)
    return out


def stable_argsort(keys) -> np.ndarray:
    keys = _i32(keys)
    out = np.empty(keys.shape[0], np.int32)
    _load().oracle_stable_argsort(keys, keys.shape[0], out)
    return out


def chunk_start(c: int, M: int, n_c: int) -> int:
    return int(_load().oracle_chunk_start(c, M, n_c))


def select(X, Y, target, permX, permY, n_c, n_ec, k, rows=None):
    """Top-k negatives of every row (or of `rows` only) over all rounds' chunk windows.

    permX: [n_r, N], permY: [n_r, C].  Returns (selected [R,k] int32 -1 padded,
    sel_score [R,k] fp32, n_cand [R] int64) for the R requested rows."""
    X, Y, target = _f32(X), _f32(Y), _i32(target)
    permX, permY = _i32(permX), _i32(permY)
    N, d = X.shape
    C = Y.shape[0]
    n_r = permX.shape[0]
    if rows is None:
        R, rows_p = N, None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R, rows_p = rows.shape[0], rows.ctypes.data_as(ctypes.c_void_p)
    sel = np.empty((R, k), np.int32)
    score = np.empty((R, k), np.float32)
    n_cand = np.empty(R, np.int64)
    _load().oracle_select(X, Y, target, N, C, d, n_c, n_ec, n_r, k, permX, permY, rows_p, R,
                          sel, score, n_cand)
    return sel, score, n_cand


def rece_loss(X, Y, target, selected):
    """(loss, row_loss [N] fp64, lse [N] fp64) of the reduced CE for a given selection."""
    X, Y, target, selected = _f32(X), _f32(Y), _i32(target), _i32(selected)
    N, d = X.shape
    k = selected.shape[1] if selected.ndim == 2 else 0
    row = np.empty(N, np.float64)
    lse = np.empty(N, np.float64)
    loss = np.zeros(1, np.float64)
    _load().oracle_rece_loss(X, Y, target, N, d, k, selected.reshape(N, k), row, lse, loss)
    return float(loss[0]), row, lse


def rece_grad(X, Y, target, selected, lse, dloss=1.0):
    """(dX [N,d], dY [C,d]) in fp64 of the reduced CE, selection held constant."""
    X, Y, target, selected = _f32(X), _f32(Y), _i32(target), _i32(selected)
    N, d = X.shape
    C = Y.shape[0]
    k = selected.shape[1]
    dX = np.empty((N, d), np.float64)
    dY = np.empty((C, d), np.float64)
    _load().oracle_rece_grad(X, Y, target, N, C, d, k, selected,
                             np.ascontiguousarray(lse, np.float64), float(dloss), dX, dY)
    return dX, dY


def rece_grad_rows(X, Y, target, rows, selected, lse, dloss=1.0):
    """dX rows of ``rece_grad`` for the row ids ``rows`` only: for each sampled row i,
    dX_i = sum over j in (z_i, then the selected entries as listed) of g_ij y_j with
    g_ij = (exp(l_ij - lse_i) - [entry is the positive]) * dloss / N, N = len(X) (RECE
    paper, equation (4) on the subset, the selection held constant).  ``selected`` [R, k]
    (-1 padded) and ``lse`` [R] follow ``rows``.  fp64 [R, d]."""
    X, Y = np.asarray(X, np.float32), np.asarray(Y, np.float32)
    N, d = X.shape
    scale = dloss / N if N else 0.0
    out = np.zeros((len(rows), d), np.float64)
    for a, i in enumerate(np.asarray(rows, np.int64)):
        js = [int(target[i])] + [int(j) for j in selected[a] if j >= 0]
        Yj = Y[js].astype(np.float64)
        g = np.exp(Yj @ X[i].astype(np.float64) - lse[a])
        g[0] -= 1.0  # the positive
        out[a] = (g * scale) @ Yj
    return out


def rece_grad_items(X, Y, target, rows, selected, lse, items, dloss=1.0):
    """dY rows of ``rece_grad`` for the item ids ``items`` only: dY_j = sum over rows i
    and entries (z_i, then the selected ones as listed) equal to j of g_ij x_i, g_ij as in
    ``rece_grad_rows``.  ``rows`` must hold every row whose positive or selection holds one
    of the items (other rows add nothing); ``selected`` [R, k] and ``lse`` [R] follow it.
    fp64 [len(items), d]."""
    X, Y = np.asarray(X, np.float32), np.asarray(Y, np.float32)
    N, d = X.shape
    scale = dloss / N if N else 0.0
    rows = np.asarray(rows, np.int64)
    sel = np.asarray(selected, np.int64).reshape(len(rows), -1)
    z = np.asarray(target, np.int64)[rows]
    out = np.zeros((len(items), d), np.float64)
    for b, j in enumerate(items):
        y = Y[j].astype(np.float64)
        n_sel = (sel == j).sum(axis=1)     # entries of the selection equal to j
        is_pos = (z == j).astype(np.int64)  # and the positive
        idx = np.nonzero(n_sel + is_pos)[0]
        if len(idx) == 0:
            continue
        Xi = X[rows[idx]].astype(np.float64)
        p = np.exp(Xi @ y - np.asarray(lse, np.float64)[idx])
        g = (p * (n_sel[idx] + is_pos[idx]) - is_pos[idx]) * scale
        out[b] = g @ Xi
    return out


def full_ce_loss(X, Y, target):
    X, Y, target = _f32(X), _f32(Y), _i32(target)
    N, d = X.shape
    row = np.empty(N, np.float64)
    lse = np.empty(N, np.float64)
    loss = np.zeros(1, np.float64)
    _load().oracle_full_ce_loss(X, Y, target, N, Y.shape[0], d, row, lse, loss)
    return float(loss[0]), row, lse


def full_ce_grad(X, Y, target, lse, dloss=1.0):
    X, Y, target = _f32(X), _f32(Y), _i32(target)
    N, d = X.shape
    C = Y.shape[0]
    dX = np.empty((N, d), np.float64)
    dY = np.empty((C, d), np.float64)
    _load().oracle_full_ce_grad(X, Y, target, N, C, d, np.ascontiguousarray(lse, np.float64),
                                float(dloss), dX, dY)
    return dX, dY


def splitmix64(state, i):
    """The i-th output (from 0) of SplitMix64 started at `state` (Steele, Lea and Flood,
    OOPSLA 2014): mix(state + (i + 1) * 0x9E3779B97F4A7C15)."""
    return int(_load().oracle_splitmix64(state & (2**64 - 1), i & (2**64 - 1)))


def draw_projections(seed, step, n_r, n_b, d):
    """Algorithm 1's random vectors B [n_r, n_b, d] (fp32) of call `step` of a run seeded
    with `seed`: standard normals by Box-Muller from the SplitMix64 stream of state
    mix(mix(seed) ^ step), elements in B's row-major order (rece_oracle.c gives every
    constant)."""
    out = np.empty(n_r * n_b * d, np.float32)
    _load().oracle_draw_projections(seed & (2**64 - 1), step & (2**64 - 1), out.size, out)
    return out.reshape(n_r, n_b, d)


def optimal_buckets(N, C, n_ec, alpha_bc):
    """RECE section 3, the paragraph before Algorithm 1: the bucket count of least peak
    memory, n_b* = sqrt(4 alpha_bc (1 + 2 n_ec) min(C, N)) with alpha_bc = n_b / n_c,
    rounded to the nearest integer (halves up) and held to [1, 4096]; n_c* = n_b* /
    alpha_bc rounded the same way and held to [1, min(N, C)]."""
    m = min(C, N)
    b = math.floor(math.sqrt(4.0 * alpha_bc * (1 + 2 * n_ec) * m) + 0.5)
    b = min(max(b, 1), 4096)
    c = min(max(math.floor(b / alpha_bc + 0.5), 1), m)
    return b, c


def memory_model_elements(N, C, n_ec, n_r, alpha_bc):
    """The same paragraph's memory complexity at n_b*, in logit elements:
    2 r sqrt(alpha_bc (1 + 2 n_ec) min(C, N)) max(C, N)."""
    return 2.0 * n_r * math.sqrt(alpha_bc * (1 + 2 * n_ec) * min(C, N)) * max(C, N)


SAMPLED_CE_MINUS = 0  # equation (2)
SAMPLED_BCE_PLUS = 1  # equation (1)


def sampled_loss(kind, X, Y, target, negatives):
    """Sampled baseline loss (section 2, eq. 2 for kind 0, eq. 1 for kind 1) over the
    given negatives [N, n] (ids < 0 are padding).  Returns (loss, row_loss, lse); lse
    is meaningful for CE- only."""
    X, Y, target, neg = _f32(X), _f32(Y), _i32(target), _i32(negatives)
    N, d = X.shape
    n = neg.shape[1] if neg.ndim == 2 else 0
    neg = neg.reshape(N, n) if N * n else np.zeros((max(N, 1), max(n, 1)), np.int32)
    row = np.empty(N, np.float64)
    lse = np.zeros(N, np.float64)
    loss = np.zeros(1, np.float64)
    _load().oracle_sampled_loss(int(kind), X, Y, target, N, d, n, neg, row, lse, loss)
    return float(loss[0]), row, lse


def sampled_grad(kind, X, Y, target, negatives, lse, dloss=1.0):
    """(dX, dY) of the sampled baseline, the negatives held constant (fp64)."""
    X, Y, target, neg = _f32(X), _f32(Y), _i32(target), _i32(negatives)
    N, d = X.shape
    C = Y.shape[0]
    n = neg.shape[1] if neg.ndim == 2 else 0
    neg = neg.reshape(N, n) if N * n else np.zeros((max(N, 1), max(n, 1)), np.int32)
    dX = np.empty((N, d), np.float64)
    dY = np.empty((C, d), np.float64)
    _load().oracle_sampled_grad(int(kind), X, Y, target, N, C, d, n, neg,
                                np.ascontiguousarray(lse, np.float64), float(dloss), dX, dY)
    return dX, dY


def _rows_arg(rows, N):
    if rows is None:
        return None, N
    r = np.ascontiguousarray(rows, np.int64)
    return r.ctypes.data_as(ctypes.c_void_p), len(r)


def window_loss(X, Y, target, permX, permY, n_c, n_ec, rows=None):
    """Algorithm 1 as printed (every window item a negative) over the rounds' stable
    orders permX [n_r, N], permY [n_r, C], duplicates across rounds corrected by
    ln(count).  rows: optional sample of row ids (outputs follow the sample, the mean is
    over it).  Returns (loss, row_loss, lse)."""
    X, Y, target = _f32(X), _f32(Y), _i32(target)
    permX, permY = _i32(permX), _i32(permY)
    N, d = X.shape
    n_r = permY.shape[0]
    keep = None if rows is None else np.ascontiguousarray(rows, np.int64)
    rp, n = _rows_arg(keep, N)
    row = np.empty(n, np.float64)
    lse = np.empty(n, np.float64)
    loss = np.zeros(1, np.float64)
    _load().oracle_window_loss(X, Y, target, N, Y.shape[0], d, n_c, n_ec, n_r,
                               permX.reshape(-1) if N else np.zeros(1, np.int32),
                               permY.reshape(-1), rp, n, row, lse, loss)
    return float(loss[0]), row, lse


def window_grad(X, Y, target, permX, permY, n_c, n_ec, lse, dloss=1.0, rows=None):
    """(dX, dY) of window_loss, the buckets and windows held constant (fp64); with a
    row sample, dX follows the sample and dY sums over it."""
    X, Y, target = _f32(X), _f32(Y), _i32(target)
    permX, permY = _i32(permX), _i32(permY)
    N, d = X.shape
    C = Y.shape[0]
    n_r = permY.shape[0]
    keep = None if rows is None else np.ascontiguousarray(rows, np.int64)
    rp, n = _rows_arg(keep, N)
    dX = np.empty((n, d), np.float64)
    dY = np.empty((C, d), np.float64)
    _load().oracle_window_grad(X, Y, target, N, C, d, n_c, n_ec, n_r,
                               permX.reshape(-1) if N else np.zeros(1, np.int32),
                               permY.reshape(-1), rp, n, np.ascontiguousarray(lse, np.float64),
                               float(dloss), dX, dY)
    return dX, dY


def rece_forward(X, Y, target, B, n_c, n_ec, k):
    """Steps 1-5 of the path given the random vectors B [n_r, n_b, d].

    Returns a dict with per-round bucket ids (bx [n_r,N], by [n_r,C]), stable orders
    (permX, permY), the selection, candidate counts, and the loss values."""
    X, Y, B = _f32(X), _f32(Y), _f32(B)
    n_r = B.shape[0]
    bx = np.stack([bucketize(X, B[r]) for r in range(n_r)]) if n_r else np.zeros((0, len(X)))
    by = np.stack([bucketize(Y, B[r]) for r in range(n_r)])
    permX = np.stack([stable_argsort(bx[r]) for r in range(n_r)])
    permY = np.stack([stable_argsort(by[r]) for r in range(n_r)])
    sel, score, n_cand = select(X, Y, target, permX, permY, n_c, n_ec, k)
    loss, row, lse = rece_loss(X, Y, target, sel)
    return dict(bx=bx, by=by, permX=permX, permY=permY, selected=sel, sel_score=score,
                n_cand=n_cand, loss=loss, row_loss=row, lse=lse)
