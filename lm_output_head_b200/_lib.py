"""ctypes declarations of the C ABI in ``include/fh.h`` (argument marshalling only).

Loading fails loudly if ``libflashhead.so`` has not been built: there is no
fallback implementation of any step.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libflashhead.so")

FH_OK = 0
FH_ERR_INVALID_ARG = 1
FH_ERR_INVALID_C2T = 2
FH_ERR_UNSUPPORTED = 3
FH_ERR_OOM = 4
FH_ERR_CUDA = 5
FH_ERR_OUT_OF_RANGE = 6
FH_ERR_TIMEOUT = 7

FH_CENTROID_BF16 = 0
FH_CENTROID_INT4_G32 = 1
FH_CENTROID_INT8_G32 = 2
FH_GREEDY = 0
FH_SAMPLE_GUMBEL = 1

FH_QUERY_WORKSPACE_BYTES = 0
FH_QUERY_LAST_UNION = 1
FH_QUERY_NUM_SMS = 2
FH_QUERY_FUSED_B1 = 3
FH_QUERY_LAST_LIST = 4
FH_QUERY_LAST_FULL = 5

# every symbol include/fh.h declares
EXPORTED = (
    "fh_create", "fh_destroy", "fh_centroid_scores", "fh_select_clusters",
    "fh_candidate_logits", "fh_decode", "fh_dense_head", "fh_get_device_status",
    "fh_status_string", "fh_set_spin_budget", "fh_query", "fh_dense_head_noalloc", "fh_speculative_verify",
    "fh_adaptive_probes", "fh_prefetch_clusters",
    # include/fh_cluster.h
    "fh_cluster_create", "fh_cluster_destroy", "fh_cluster_normalize", "fh_cluster_seed",
    "fh_cluster_gather", "fh_cluster_similarities", "fh_cluster_assign", "fh_cluster_update",
    "fh_cluster_build", "fh_cluster_get_device_status",
)

FH_C2T_INT32 = 0
FH_C2T_UINT16 = 1

FH_NOALLOC_MAX_ROWS = 64


class HeadDesc(ctypes.Structure):
    _fields_ = [
        ("v", ctypes.c_int32), ("d", ctypes.c_int32), ("c", ctypes.c_int32), ("b", ctypes.c_int32),
        ("E", ctypes.c_void_p), ("C", ctypes.c_void_p), ("C_q", ctypes.c_void_p),
        ("C_scales", ctypes.c_void_p), ("C2T", ctypes.c_void_p),
        ("fmt", ctypes.c_int32), ("max_batch", ctypes.c_int32), ("max_probes", ctypes.c_int32),
        ("c2t_format", ctypes.c_int32),
    ]


class FlashHeadError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m lm_output_head_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    lib.fh_create.argtypes = [ctypes.POINTER(HeadDesc), vp, ctypes.POINTER(vp)]
    lib.fh_create.restype = ctypes.c_int
    lib.fh_destroy.argtypes = [vp]
    lib.fh_destroy.restype = None
    lib.fh_centroid_scores.argtypes = [vp, vp, i32, vp, vp]
    lib.fh_centroid_scores.restype = ctypes.c_int
    lib.fh_select_clusters.argtypes = [vp, vp, i32, i32, i32, f32, vp, vp, vp]
    lib.fh_select_clusters.restype = ctypes.c_int
    lib.fh_candidate_logits.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp]
    lib.fh_candidate_logits.restype = ctypes.c_int
    lib.fh_decode.argtypes = [vp, vp, i32, i32, i32, f32, vp, vp, vp, vp, vp, vp]
    lib.fh_decode.restype = ctypes.c_int
    lib.fh_dense_head.argtypes = [vp, vp, i32, vp, vp, vp]
    lib.fh_dense_head.restype = ctypes.c_int
    lib.fh_dense_head_noalloc.argtypes = [vp, i32, i32, vp, i32, vp, vp, vp]
    lib.fh_dense_head_noalloc.restype = ctypes.c_int
    lib.fh_get_device_status.argtypes = [vp, vp]
    lib.fh_get_device_status.restype = ctypes.c_int
    lib.fh_status_string.argtypes = [ctypes.c_int]
    lib.fh_status_string.restype = ctypes.c_char_p
    lib.fh_set_spin_budget.argtypes = [vp, ctypes.c_int64]
    lib.fh_set_spin_budget.restype = ctypes.c_int
    lib.fh_query.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_int64)]
    lib.fh_query.restype = ctypes.c_int
    lib.fh_speculative_verify.argtypes = [vp, vp, vp, i32, i32, vp, f32, vp, vp, vp, vp]
    lib.fh_speculative_verify.restype = ctypes.c_int
    lib.fh_adaptive_probes.argtypes = [vp, vp, i32, f32, i32, i32, f32, vp, vp]
    lib.fh_adaptive_probes.restype = ctypes.c_int
    lib.fh_prefetch_clusters.argtypes = [vp, vp, i32, vp]
    lib.fh_prefetch_clusters.restype = ctypes.c_int
    pi32 = ctypes.POINTER(ctypes.c_int32)
    lib.fh_cluster_create.argtypes = [i32, i32, i32, vp, ctypes.POINTER(vp)]
    lib.fh_cluster_destroy.argtypes = [vp]
    lib.fh_cluster_destroy.restype = None
    lib.fh_cluster_normalize.argtypes = [vp, vp, vp, vp]
    lib.fh_cluster_seed.argtypes = [vp, vp, vp, vp, vp]
    lib.fh_cluster_gather.argtypes = [vp, vp, vp, vp, vp]
    lib.fh_cluster_similarities.argtypes = [vp, vp, vp, vp, vp]
    lib.fh_cluster_assign.argtypes = [vp, vp, vp, vp, pi32, vp]
    lib.fh_cluster_update.argtypes = [vp, vp, vp, vp, vp]
    lib.fh_cluster_build.argtypes = [vp, vp, vp, vp, i32, vp, vp, pi32, vp]
    lib.fh_cluster_get_device_status.argtypes = [vp, vp]
    for name in ("fh_cluster_create", "fh_cluster_normalize", "fh_cluster_seed", "fh_cluster_gather",
                 "fh_cluster_similarities", "fh_cluster_assign", "fh_cluster_update", "fh_cluster_build",
                 "fh_cluster_get_device_status"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().fh_status_string(int(status)).decode()
