"""ctypes loader for libgmm_fp8.so: argument marshalling only.

The library sits next to this file (built in-tree by ``build.py``).  Loading
fails loudly when it is missing: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgmm_fp8.so")

# enums of include/gmm_fp8.h
GMM_OK = 0
STATUS_NAMES = {0: "GMM_OK", 1: "GMM_ERR_INVALID_ARG", 2: "GMM_ERR_SHAPE", 3: "GMM_ERR_ALIGNMENT",
                4: "GMM_ERR_SCALE", 5: "GMM_ERR_UNSUPPORTED", 6: "GMM_ERR_CUDA", 7: "GMM_ERR_GROUP_SIZES",
                8: "GMM_ERR_TIMEOUT", 9: "GMM_ERR_WORKSPACE"}
Q_NONE, Q_STATIC, Q_DYNAMIC = 0, 1, 2
DT_BF16, DT_F32, DT_E4M3 = 0, 1, 2
OP_FWD, OP_DLHS, OP_DRHS, OP_BWD = 0, 1, 2, 3
DEV_GROUP_SIZES, DEV_SCALE, DEV_TIMEOUT = 1, 2, 4
TILES_AUTO, TILES_ONE_CTA, TILES_CTA_PAIRS, TILES_CTA_PAIRS_NARROW = 0, 1, 2, 3

# every symbol include/gmm_fp8.h declares
EXPORTS = ["gmm_workspace_bytes", "gmm_chunk_capacity", "gmm_quantize_rhs", "gmm_quantize", "gmm_fwd",
           "gmm_dlhs", "tgmm_drhs", "gmm_read_device_status", "gmm_selftest_timeout", "gmm_set_wait_limit_ns",
           "gmm_status_string", "gmm_last_launch_count", "gmm_profile_enable", "gmm_profile_collect",
           "gmm_fwd_noalloc", "gmm_fwd_swiglu", "gmm_quantize_rhs_blocks", "gmm_gather_rows",
           "gmm_combine_rows", "gmm_backward", "gmm_gather_scale_rows", "gmm_fwd_keep_lhs",
           "gmm_fwd_noalloc_status", "gmm_set_tiles", "gmm_ep_local_order"]


class Operand(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int), ("scale", ctypes.c_void_p),
                ("rule", ctypes.c_int)]


class ProfileEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_double)]


_lib = None


def lib():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with moe_fp8_grouped_b200.build.build() "
                           "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64
    st = ctypes.c_int
    L.gmm_workspace_bytes.argtypes = [ctypes.c_int, i64, i64, i64, i32]
    L.gmm_workspace_bytes.restype = sz
    L.gmm_chunk_capacity.argtypes = [i64, i32]
    L.gmm_chunk_capacity.restype = i64
    L.gmm_quantize_rhs.argtypes = [vp, i32, i64, i64, ctypes.c_int, vp, vp, vp]
    L.gmm_quantize_rhs.restype = st
    L.gmm_quantize.argtypes = [vp, i64, i64, ctypes.c_int, ctypes.c_int, vp, vp, i32, vp, vp, vp, vp, sz, vp]
    L.gmm_quantize.restype = st
    L.gmm_fwd.argtypes = [Operand, Operand, ctypes.c_int, vp, i32, i64, i64, i64, vp, ctypes.c_int, vp, sz, vp]
    L.gmm_fwd.restype = st
    L.gmm_fwd_swiglu.argtypes = L.gmm_fwd.argtypes
    L.gmm_fwd_keep_lhs.argtypes = [Operand, Operand, ctypes.c_int, vp, i32, i64, i64, i64, vp, ctypes.c_int, vp, sz,
                                   vp, vp, vp]
    L.gmm_fwd_keep_lhs.restype = st
    L.gmm_quantize_rhs_blocks.argtypes = [vp, i32, i64, i64, ctypes.c_int, vp, vp, vp]
    L.gmm_quantize_rhs_blocks.restype = st
    L.gmm_backward.argtypes = [Operand, Operand, Operand, ctypes.c_int, vp, i32, i64, i64, i64, vp, ctypes.c_int,
                               vp, ctypes.c_int, vp, sz, vp]
    L.gmm_backward.restype = st
    L.gmm_gather_rows.argtypes = [vp, vp, i64, i64, i64, vp, vp]
    L.gmm_gather_scale_rows.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp]
    L.gmm_gather_scale_rows.restype = st
    L.gmm_gather_rows.restype = st
    L.gmm_combine_rows.argtypes = [vp, i64, vp, vp, i64, i32, i64, vp, ctypes.c_int, vp]
    L.gmm_combine_rows.restype = st
    L.gmm_ep_local_order.argtypes = [vp, i32, i32, i64, vp, vp, vp, vp]
    L.gmm_ep_local_order.restype = st
    L.gmm_fwd_swiglu.restype = st
    L.gmm_fwd_noalloc.argtypes = [Operand, Operand, ctypes.c_int, vp, i32, i64, i64, i64, vp, ctypes.c_int, vp]
    L.gmm_fwd_noalloc.restype = st
    L.gmm_fwd_noalloc_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), vp]
    L.gmm_fwd_noalloc_status.restype = st
    L.gmm_dlhs.argtypes = L.gmm_fwd.argtypes
    L.gmm_dlhs.restype = st
    L.tgmm_drhs.argtypes = [Operand, Operand, vp, i32, i64, i64, i64, vp, ctypes.c_int, vp, sz, vp]
    L.tgmm_drhs.restype = st
    L.gmm_read_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), vp]
    L.gmm_read_device_status.restype = st
    L.gmm_selftest_timeout.argtypes = [vp, u64, vp]
    L.gmm_selftest_timeout.restype = st
    L.gmm_set_wait_limit_ns.argtypes = [u64]
    L.gmm_set_wait_limit_ns.restype = None
    L.gmm_set_tiles.argtypes = [i32]
    L.gmm_set_tiles.restype = st
    L.gmm_status_string.argtypes = [ctypes.c_int]
    L.gmm_status_string.restype = ctypes.c_char_p
    L.gmm_last_launch_count.argtypes = []
    L.gmm_last_launch_count.restype = i32
    L.gmm_profile_enable.argtypes = [ctypes.c_int]
    L.gmm_profile_enable.restype = None
    L.gmm_profile_collect.argtypes = [ctypes.POINTER(ProfileEntry), i32]
    L.gmm_profile_collect.restype = i32
    _lib = L
    return L
