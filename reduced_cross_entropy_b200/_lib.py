"""ctypes view of the C ABI in ``include/rece.h`` (``librece_b200.so``).

Nothing here computes: it declares the entry points and loads the in-tree library.
A missing library raises at first use -- there is no fallback implementation.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "librece_b200.so")

RECE_OK = 0
STATUS_NAMES = {0: "RECE_OK", 1: "RECE_ERR_INVALID_ARG", 2: "RECE_ERR_UNSUPPORTED",
                3: "RECE_ERR_WORKSPACE", 4: "RECE_ERR_CUDA", 5: "RECE_ERR_DEVICE_INPUT",
                6: "RECE_ERR_TIMEOUT", 7: "RECE_ERR_NO_DEVICE"}
MODE_FP32_EXACT = 0
MODE_BF16 = 1
FLAG_FMA_SCORES = 0x1
DEVICE_BAD_TARGET = 0x1
DEVICE_TIMEOUT = 0x2
DEVICE_INEXACT = 0x4
PATH_TENSOR_CORES = 0x1
PATH_DX_TENSORS = 0x2
PATH_STORED_SCORES = 0x4
PATH_ALL_NEGATIVES = 0x8
PATH_DY_TENSORS = 0x10
PATH_DX_PARTS = 0x20
PATH_SAMPLED_SELECT = 0x40
PATH_WINDOW_FMA = 0x80  # with PATH_ALL_NEGATIVES: window sums on the CUDA cores
FLAG_ALL_NEGATIVES = 0x2  # Algorithm 1 as printed: every window item a negative

# every symbol include/rece.h declares
EXPORTS = (
    "rece_plan_create", "rece_plan_destroy", "rece_plan_workspace_size",
    "rece_plan_workspace_layout", "rece_bucketize_sort", "rece_loss_fwd", "rece_loss_bwd",
    "rece_full_ce_workspace_size", "rece_full_ce_fwd", "rece_full_ce_bwd",
    "rece_get_device_status", "rece_status_string", "rece_last_error_string",
    "rece_plan_set_stage_events", "rece_kernel_launch_count", "rece_bucket_sort_static",
    "rece_plan_paths", "rece_sampled_workspace_size", "rece_sampled_fwd", "rece_sampled_bwd",
    "rece_optimal_buckets", "rece_memory_model_elements", "rece_plan_get_config",
    "rece_draw_projections",
)
SAMPLED_CE_MINUS = 0  # RECE section 2, equation (2)
SAMPLED_BCE_PLUS = 1  # RECE section 2, equation (1)
STAGES = ("bucketize", "sort", "select", "merge_loss", "mean", "bwd_rows", "bwd_sort",
          "bwd_items")


class Config(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("C", ctypes.c_int64), ("d", ctypes.c_int32),
                ("n_b", ctypes.c_int32), ("n_c", ctypes.c_int32), ("n_ec", ctypes.c_int32),
                ("n_r", ctypes.c_int32), ("k", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("status", "bucket_x", "bucket_y", "perm_x",
                                               "perm_y", "bucket_start_y",
                                               "bucket_start_stride")]


class ReceError(RuntimeError):
    def __init__(self, status, where, detail=""):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}"
                         + (f" ({detail})" if detail else ""))


_lib = None


def lib():
    """The loaded library (loaded once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m reduced_cross_entropy_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i64, i32, u32 = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int32,
                             ctypes.c_uint32)
    st = ctypes.c_int
    sig = {
        "rece_plan_create": ([ctypes.POINTER(Config), ctypes.POINTER(vp)], st),
        "rece_plan_destroy": ([vp], None),
        "rece_plan_workspace_size": ([vp, ctypes.POINTER(sz)], st),
        "rece_plan_get_config": ([vp, ctypes.POINTER(Config)], st),
        "rece_plan_workspace_layout": ([vp, ctypes.POINTER(WorkspaceLayout)], st),
        "rece_plan_paths": ([vp, ctypes.POINTER(ctypes.c_uint32)], st),
        "rece_bucketize_sort": ([vp, vp, vp, vp, vp, sz, vp], st),
        "rece_draw_projections": ([vp, ctypes.c_uint64, ctypes.c_uint64, vp, vp], st),
        "rece_loss_fwd": ([vp, vp, vp, vp, vp, sz, vp, vp, vp, vp, vp, vp], st),
        "rece_loss_bwd": ([vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp], st),
        "rece_full_ce_workspace_size": ([i64, i64, i32, i32, ctypes.POINTER(sz)], st),
        "rece_full_ce_fwd": ([i64, i64, i32, i32, vp, vp, vp, vp, sz, vp, vp, vp, vp], st),
        "rece_full_ce_bwd": ([i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp], st),
        "rece_get_device_status": ([vp, ctypes.POINTER(u32), vp], st),
        "rece_status_string": ([st], ctypes.c_char_p),
        "rece_last_error_string": ([], ctypes.c_char_p),
        "rece_plan_set_stage_events": ([vp, ctypes.POINTER(vp)], st),
        "rece_kernel_launch_count": ([], ctypes.c_uint64),
        "rece_bucket_sort_static": ([vp, i64, i32, vp, vp, vp], st),
        "rece_sampled_workspace_size": ([i32, i64, i64, i32, i32, i32, ctypes.POINTER(sz)], st),
        "rece_optimal_buckets": ([i64, i64, i32, ctypes.c_double, ctypes.POINTER(i32),
                                  ctypes.POINTER(i32)], st),
        "rece_memory_model_elements": ([i64, i64, i32, i32, ctypes.c_double,
                                        ctypes.POINTER(ctypes.c_double)], st),
        "rece_sampled_fwd": ([i32, i64, i64, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp, vp,
                              vp, vp], st),
        "rece_sampled_bwd": ([i32, i64, i64, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                              vp, vp, vp], st),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def check(status, where):
    if status != RECE_OK:
        detail = lib().rece_last_error_string().decode(errors="replace")
        raise ReceError(status, where, detail)
