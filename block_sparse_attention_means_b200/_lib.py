"""ctypes declaration of the libpark C ABI (include/park.h).  Marshalling only."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpark.so")

PARK_OK = 0
PARK_ERR_INVALID_ARG = 1
PARK_ERR_UNSUPPORTED = 2
PARK_ERR_WORKSPACE = 3
PARK_ERR_CUDA = 4
PARK_ERR_RANGE = 5
PARK_ERR_TIMEOUT = 6

PARK_BF16 = 0
PARK_F32 = 1

PARK_FLAG_WARM_START_Q = 0x1
PARK_FLAG_WARM_START_K = 0x2
PARK_FLAG_NO_QRKC = 0x4
PARK_FLAG_CENTROID_QUERY = 0x8
PARK_FLAG_TOPK = 0x10
PARK_FLAG_SIZE_PRIOR = 0x20
PARK_FLAG_SIP = 0x40
PARK_FLAG_MERGE_Q = 0x80
PARK_FLAG_LOCAL_WINDOW = 0x100
PARK_FLAG_NO_TILE_PACKING = 0x200

PARK_CNT_Q_RECHECK = 0
PARK_CNT_K_RECHECK = 1
PARK_CNT_FULL_RESCORE = 2
PARK_CNT_PAMA_RECHECK = 3
PARK_CNT_KEPT_BLOCKS = 4
PARK_CNT_KEPT_PAIRS = 5
PARK_CNT_WORK_ITEMS = 6
PARK_CNT_KEY_TILES = 7
PARK_NUM_COUNTERS = 8

# Every symbol include/park.h declares (checked by the CPU tests).
EXPORTS = ("park_workspace_size", "park_retrieve", "park_sparse_attn", "park_layer", "park_status_string",
           "park_launch_count", "park_version", "park_profile_enable", "park_profile_collect",
           "park_qrkc_metric_static", "park_set_wait_limit_ns")


class ParkShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("Hg", ctypes.c_int),
                ("W", ctypes.c_int), ("n_text", ctypes.c_int), ("D", ctypes.c_int), ("dtype", ctypes.c_int)]


class ParkRetrieval(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint32),
                ("q_labels", ctypes.c_void_p), ("k_labels", ctypes.c_void_p),
                ("q_perm", ctypes.c_void_p), ("k_perm", ctypes.c_void_p),
                ("q_offsets", ctypes.c_void_p), ("k_offsets", ctypes.c_void_p),
                ("q_centroids", ctypes.c_void_p), ("k_centroids", ctypes.c_void_p),
                ("importance", ctypes.c_void_p), ("mask", ctypes.c_void_p),
                ("kept_ptr", ctypes.c_void_p), ("kept_idx", ctypes.c_void_p),
                ("metric", ctypes.c_void_p), ("importance_bound", ctypes.c_void_p),
                ("counters", ctypes.c_void_p), ("status", ctypes.c_void_p),
                ("sip_uniform", ctypes.c_void_p), ("block_weight", ctypes.c_void_p),
                ("window_t", ctypes.c_int32), ("window_h", ctypes.c_int32), ("window_w", ctypes.c_int32),
                ("merge_rounds", ctypes.c_int32)]


class ParkKernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("total_ms", ctypes.c_double), ("launches", ctypes.c_int64)]


class ParkError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} (code {code})")
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Load libpark.so (built in-tree).  Raises if it is missing: there is no
    fallback implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m block_sparse_attention_means_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    shp = ctypes.POINTER(ParkShape)
    ret = ctypes.POINTER(ParkRetrieval)
    lib.park_workspace_size.argtypes = [shp, i32, i32, ctypes.POINTER(sz)]
    lib.park_retrieve.argtypes = [vp, vp, shp, i32, i32, f32, i32, ret, vp, sz, vp]
    lib.park_sparse_attn.argtypes = [vp, vp, vp, shp, i32, i32, ret, vp, vp, sz, vp]
    lib.park_layer.argtypes = [vp, vp, vp, shp, i32, i32, f32, i32, vp, ret, vp, sz, vp]
    for f in ("park_workspace_size", "park_retrieve", "park_sparse_attn", "park_layer"):
        getattr(lib, f).restype = i32
    lib.park_status_string.argtypes = [i32]
    lib.park_status_string.restype = ctypes.c_char_p
    lib.park_launch_count.argtypes = []
    lib.park_launch_count.restype = ctypes.c_uint64
    lib.park_version.argtypes = []
    lib.park_version.restype = i32
    lib.park_profile_enable.argtypes = [i32]
    lib.park_profile_enable.restype = i32
    lib.park_profile_collect.argtypes = [ctypes.POINTER(ParkKernelTime), i32, ctypes.POINTER(i32)]
    lib.park_profile_collect.restype = i32
    lib.park_qrkc_metric_static.argtypes = [vp, shp, vp, vp]
    lib.park_qrkc_metric_static.restype = i32
    lib.park_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.park_set_wait_limit_ns.restype = i32
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().park_status_string(int(code)).decode()


def check(code: int, what: str) -> None:
    if code != PARK_OK:
        raise ParkError(code, what)
