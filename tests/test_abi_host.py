"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/rece.h declares, validates configs and sizes its workspace."""
import ctypes
import os
import re

import pytest

from reduced_cross_entropy_b200 import _lib, build
from reduced_cross_entropy_b200.ops import Plan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build.build()
    return _lib.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "rece.h")).read()
    return sorted(set(re.findall(r"RECE_API[^;(]*?\b(rece_\w+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 13
    assert sorted(_lib.EXPORTS) == names
    L = _lib.lib()
    for n in names:
        assert getattr(L, n) is not None


def test_status_strings():
    L = _lib.lib()
    for code, name in _lib.STATUS_NAMES.items():
        assert L.rece_status_string(code).decode() == name


def cfg(**kw):
    base = dict(N=256, C=4096, d=64, n_b=16, n_c=8, n_ec=1, n_r=1, k=32, mode=0, flags=0)
    base.update(kw)
    return _lib.Config(**base)


def create(c):
    h = ctypes.c_void_p()
    s = _lib.lib().rece_plan_create(ctypes.byref(c), ctypes.byref(h))
    if s == 0:
        _lib.lib().rece_plan_destroy(h)
    return s


@pytest.mark.parametrize("bad", [
    dict(N=-1), dict(C=0), dict(d=0), dict(n_b=0), dict(n_b=4097), dict(n_r=0), dict(n_r=9),
    dict(k=0), dict(k=4097), dict(n_ec=-1), dict(n_c=0), dict(n_c=257), dict(C=100, n_c=101),
    dict(n_b=0, n_c=0, N=-1), dict(n_b=0, n_c=0, C=0), dict(n_b=0, n_c=0, n_ec=-1),
    dict(mode=2), dict(flags=0x80),
])
def test_invalid_configs_rejected(bad):
    assert create(cfg(**bad)) == 1
    assert _lib.lib().rece_last_error_string().decode() != ""


def test_unsupported_sizes():
    assert create(cfg(n_r=4, k=4096)) == 2           # merge buffer bound n_r * k <= 8192
    assert create(cfg(N=1 << 21, k=1024, n_c=8)) == 2  # 32-bit pair indexing


def test_valid_edge_configs():
    assert create(cfg()) == 0
    assert create(cfg(N=0, n_c=8)) == 0                 # empty batch
    assert create(cfg(C=1, N=5, n_c=1, k=1)) == 0       # single item
    assert create(cfg(n_b=1, n_c=1, k=4095)) == 0       # full-CE reduction
    assert create(cfg(n_b=4096)) == 0


def test_null_arguments():
    L = _lib.lib()
    assert L.rece_plan_create(None, None) == 1
    assert L.rece_plan_workspace_size(None, None) == 1
    assert L.rece_bucketize_sort(None, None, None, None, None, 0, None) == 1
    assert L.rece_draw_projections(None, 0, 0, None, None) == 1
    p = Plan(N=256, C=4096, d=64, n_b=16, n_c=8, n_ec=1, n_r=1, k=32)
    assert L.rece_draw_projections(p._h, 0, 0, None, None) == 1  # NULL B


def test_workspace_size_and_layout():
    for w in [dict(), dict(N=25600, C=100000, n_b=256, n_c=64, n_r=2, k=256, mode=1),
              dict(N=0, n_c=8)]:
        p = Plan(**{k: v for k, v in {**dict(N=256, C=4096, d=64, n_b=16, n_c=8, n_ec=1, n_r=1,
                                             k=32), **w}.items() if k != "mode"},
                 mode=w.get("mode", 0))
        c = p.cfg
        lay = p.layout
        assert lay.status == 0
        offs = [lay.bucket_x, lay.bucket_y, lay.perm_x, lay.perm_y, lay.bucket_start_y]
        assert all(o % 256 == 0 for o in offs)
        # the arrays the caller may read after rece_bucketize_sort do not overlap
        spans = sorted([(lay.bucket_x, 4 * c.n_r * c.N), (lay.bucket_y, 4 * c.n_r * c.C),
                        (lay.perm_x, 4 * c.n_r * c.N), (lay.perm_y, 4 * c.n_r * c.C),
                        (lay.bucket_start_y, 4 * c.n_r * lay.bucket_start_stride)])
        for (a, na), (b, _) in zip(spans, spans[1:]):
            assert a + na <= b
        assert spans[-1][0] + spans[-1][1] <= p.workspace_bytes
        lists = 8 * c.n_r * c.N * c.k
        pairs = 5 * 4 * c.N * (c.k + 1)
        assert p.workspace_bytes >= max(lists, pairs)
        assert lay.bucket_start_stride == (1 << (c.n_b - 1).bit_length()) + 1


def test_full_ce_workspace_size():
    size = ctypes.c_size_t()
    assert _lib.lib().rece_full_ce_workspace_size(100, 10, 8, 0, ctypes.byref(size)) == 0
    assert size.value >= 4 + 400
    assert _lib.lib().rece_full_ce_workspace_size(100, 0, 8, 0, ctypes.byref(size)) == 1


def test_calls_reject_small_workspace_without_gpu():
    p = Plan(N=256, C=4096, d=64, n_b=16, n_c=8, n_r=1, k=32, mode="fp32")
    L = _lib.lib()
    ws = ctypes.c_void_p(256)  # never dereferenced: rejected on the host first
    s = L.rece_bucketize_sort(p._h, ctypes.c_void_p(512), ctypes.c_void_p(512),
                              ctypes.c_void_p(512), ws, 16, None)
    assert s == 3


def test_calls_reject_misaligned_matrices_without_gpu():
    # the kernels use 16-byte vector loads, stores and bulk copies on X, Y, B, dX, dY
    p = Plan(N=256, C=4096, d=64, n_b=16, n_c=8, n_r=1, k=32, mode="fp32")
    L = _lib.lib()
    ws = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected on the host first
    ok, bad = ctypes.c_void_p(1 << 16), ctypes.c_void_p((1 << 16) + 8)
    n = p.workspace_bytes
    assert L.rece_bucketize_sort(p._h, ok, bad, ok, ws, n, None) == 1
    assert L.rece_bucketize_sort(p._h, bad, ok, ok, ws, n, None) == 1
    assert b"16-byte aligned" in L.rece_last_error_string()
    args = [ok] * 7  # X, Y, targets, selected, lse, logits, dloss
    assert L.rece_loss_bwd(p._h, *args, ws, n, ok, bad, None) == 1
    assert L.rece_loss_bwd(p._h, bad, *args[1:], ws, n, ok, ok, None) == 1


def test_plan_paths_follow_the_shape():
    """rece_plan_paths: which kernels a plan runs (decided on the host, no GPU needed)."""
    TC, DX, SC = _lib.PATH_TENSOR_CORES, _lib.PATH_DX_TENSORS, _lib.PATH_STORED_SCORES
    DY, PARTS = _lib.PATH_DY_TENSORS, _lib.PATH_DX_PARTS
    from reduced_cross_entropy_b200 import synth
    W = synth.WORKLOADS

    def paths(w, **over):
        w = w.scaled(w.N, w.C, **over) if over else w
        return Plan(w.N, w.C, w.d, w.n_b, w.n_c, w.n_ec, w.n_r, w.k, mode=w.dtype).paths

    assert paths(W["tiny"]) == 0                      # fp32 exact mode: fmaf kernels
    assert paths(W["sasrec"]) == TC                   # catalogue in L2: gathered dX
    # 256 MB catalogue: dX and dY on tcgen05; 400 row tiles a round, two CTAs an SM: both
    # rounds in one launch (parts summed in order) fill the waves better than a launch a round
    assert paths(W["large"]) == TC | DX | DY | PARTS
    # d = 4096: stored scores, dY on tcgen05; 1024 work items a round: a launch a round
    assert paths(W["lm"]) == TC | DX | SC | DY
    # d = 256: the selection's threshold from a sample of the window, one streaming pass
    assert paths(W["very_large"]) == TC | DX | DY | PARTS | _lib.PATH_SAMPLED_SELECT
    # catalogues beyond half of L2 at small d: dX on tcgen05, dY too from d = 128 on
    big = W["sasrec"].scaled(25_600, 600_000)
    assert paths(big) & (DX | DY) == DX                 # d = 64: dY by the pair sort
    assert paths(big, d=128) & (DX | DY) == DX | DY
    assert paths(W["sasrec"], d=48) == 0              # d not a multiple of 64
    p = Plan(256, 4096, 64, 16, 8, 1, 1, 32, mode="bf16", flags=_lib.FLAG_FMA_SCORES)
    assert p.paths == 0                               # fmaf scores on request


def test_optimal_buckets_and_memory_model_match_the_oracle():
    import oracle
    from reduced_cross_entropy_b200 import ops
    for N, C, n_ec, n_r, a in [(25600, 100000, 1, 2, 4.0), (51200, 10 ** 6, 1, 2, 1.0),
                               (300, 200, 0, 1, 0.5), (16384, 128000, 2, 3, 2.0),
                               (7, 10 ** 9, 2, 1, 2.0), (10 ** 9, 10 ** 9, 3, 1, 4.0),
                               (1, 1, 0, 1, 1.0), (2500, 3000, 0, 1, 0.25)]:
        assert ops.optimal_buckets(N, C, n_ec, a) == oracle.optimal_buckets(N, C, n_ec, a)
        assert ops.memory_model_elements(N, C, n_ec, n_r, a) == pytest.approx(
            oracle.memory_model_elements(N, C, n_ec, n_r, a), rel=1e-12)
    L = _lib.lib()
    nb, nc, v = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_double()
    assert L.rece_optimal_buckets(10, 10, 0, 0.0, ctypes.byref(nb), ctypes.byref(nc)) == 1
    assert L.rece_optimal_buckets(0, 10, 0, 1.0, ctypes.byref(nb), ctypes.byref(nc)) == 1
    assert L.rece_memory_model_elements(10, 10, -1, 1, 1.0, ctypes.byref(v)) == 1


def test_sampled_workspace_and_validation():
    from reduced_cross_entropy_b200 import ops
    small = ops.sampled_workspace_bytes("ce_minus", 1000, 5000, 64, 10, "bf16")
    large = ops.sampled_workspace_bytes("ce_minus", 1000, 5000, 64, 100, "bf16")
    assert 0 < small < large
    assert ops.sampled_workspace_bytes("bce_plus", 0, 5000, 64, 10, "fp32") > 0
    L = _lib.lib()
    sz = ctypes.c_size_t()
    assert L.rece_sampled_workspace_size(2, 10, 10, 8, 1, 0, ctypes.byref(sz)) == 1  # kind
    assert L.rece_sampled_workspace_size(0, 10, 10, 8, -1, 0, ctypes.byref(sz)) == 1  # n
    assert L.rece_sampled_workspace_size(0, 10, 10, 8, 1, 7, ctypes.byref(sz)) == 1  # mode
    assert L.rece_sampled_workspace_size(0, 10, 10, 50000, 1000, 0, ctypes.byref(sz)) == 2
    assert L.rece_sampled_workspace_size(0, 2 ** 20, 10, 8, 4096, 0, ctypes.byref(sz)) == 2
    # a workspace smaller than asked for is refused before anything is launched
    one = ctypes.c_void_p(256)
    assert L.rece_sampled_fwd(0, 10, 10, 8, 1, 0, one, one, one, one, one, 16, one, None,
                              None, one, None) == 3


def test_all_negatives_mode_support():
    """Algorithm 1 as printed: window sums on tcgen05 for bf16 with d a multiple of 64 up
    to 256, on the CUDA cores (fmaf chains) for every other shape and mode."""
    flags = _lib.FLAG_ALL_NEGATIVES
    TC, AN, FMA = _lib.PATH_TENSOR_CORES, _lib.PATH_ALL_NEGATIVES, _lib.PATH_WINDOW_FMA
    p = Plan(1000, 5000, 128, 16, 8, 1, 2, 8, mode="bf16", flags=flags)
    assert p.paths == TC | AN
    assert p.workspace_bytes > 0

    def paths(**over):
        kw = dict(N=1000, C=5000, d=128, n_b=16, n_c=8, n_ec=1, n_r=2, k=8, mode="bf16")
        kw.update(over)
        return Plan(kw["N"], kw["C"], kw["d"], kw["n_b"], kw["n_c"], kw["n_ec"], kw["n_r"],
                    kw["k"], mode=kw["mode"], flags=kw.get("flags", flags)).paths

    assert paths(mode="fp32") == AN | FMA                   # fp32 exact mode
    assert paths(d=512) == TC | AN | FMA                    # bucketing on tcgen05 only
    assert paths(d=4096, N=16_384, C=128_000, n_b=512, n_c=128) == TC | AN | FMA  # LM shape
    assert paths(d=96) == AN | FMA                          # d not a multiple of 64
    assert paths(flags=flags | _lib.FLAG_FMA_SCORES) == AN | FMA
    # the CUDA-core mode keeps no sorted copies: a smaller workspace than the tcgen05 one
    a = Plan(1000, 5000, 128, 16, 8, 1, 2, 8, mode="bf16", flags=flags)
    b = Plan(1000, 5000, 128, 16, 8, 1, 2, 8, mode="bf16", flags=flags | _lib.FLAG_FMA_SCORES)
    assert b.workspace_bytes < a.workspace_bytes


@pytest.mark.parametrize("N,C,n_ec", [(256, 4096, 1), (25_600, 100_000, 1),
                                      (65_536, 4_000_000, 2), (3, 100, 0), (0, 50, 1),
                                      (10**6, 2 * 10**6, 8)])
def test_zero_buckets_and_chunks_mean_the_pages_optimum(N, C, n_ec):
    """n_b = n_c = 0: n_b* = sqrt(4 alpha_bc (1 + 2 n_ec) min(C, N)) at alpha_bc = 1, rounded
    to the nearest integer, n_b held to [1, 4096] and n_c = n_b to [1, min(N, C)] (RECE
    section 3, the paragraph before Algorithm 1; section 5 for alpha_bc = 1)."""
    import math
    p = Plan(N, C, 64, 0, 0, n_ec, 1, 8, mode="fp32")
    m = min(N, C)
    want = min(max(int(math.floor(math.sqrt(4 * (1 + 2 * n_ec) * m) + 0.5)), 1), 4096)
    want_c = min(max(want, 1), max(m, 1))
    assert (p.n_b, p.n_c) == (want, want_c)
    assert (p.N, p.C, p.n_ec) == (N, C, n_ec)
    # the same numbers as the helper the library exports
    nb, nc = ctypes.c_int32(), ctypes.c_int32()
    if N > 0:
        assert _lib.lib().rece_optimal_buckets(N, C, n_ec, 1.0, ctypes.byref(nb),
                                               ctypes.byref(nc)) == 0
        assert (nb.value, nc.value) == (p.n_b, p.n_c)
    # an explicit plan with those numbers is the same plan
    q = Plan(N, C, 64, p.n_b, p.n_c, n_ec, 1, 8, mode="fp32")
    assert q.workspace_bytes == p.workspace_bytes


def test_zero_buckets_needs_zero_chunks_too():
    assert create(cfg(n_b=0, n_c=8)) == 1
    assert create(cfg(n_b=16, n_c=0)) == 1
    assert b"both" in _lib.lib().rece_last_error_string()
