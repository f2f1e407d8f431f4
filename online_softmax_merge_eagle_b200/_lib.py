"""ctypes view of include/eagleattn.h (loaded from the in-tree libeagleattn.so).

Nothing here computes: it mirrors the C structs and prototypes.  Loading
fails loudly when the library has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libeagleattn.so")

ABI_VERSION = 4

OK = 0
STATUS = {
    0: "EAGLE_ATTN_OK", -1: "EAGLE_ATTN_ERR_NULL", -2: "EAGLE_ATTN_ERR_ABI",
    -3: "EAGLE_ATTN_ERR_DTYPE", -4: "EAGLE_ATTN_ERR_SHAPE", -5: "EAGLE_ATTN_ERR_STRIDE",
    -6: "EAGLE_ATTN_ERR_ALIGN", -7: "EAGLE_ATTN_ERR_VARLEN", -8: "EAGLE_ATTN_ERR_WORKSPACE",
    -9: "EAGLE_ATTN_ERR_UNSUPPORTED", -10: "EAGLE_ATTN_ERR_CUDA", -11: "EAGLE_ATTN_ERR_DEVICE",
    -12: "EAGLE_ATTN_ERR_SCRATCH_LIMIT",
}
NOALLOC_SCRATCH_BYTES = 32 << 20
DEV_STATUS = {0: "EAGLE_ATTN_DEV_OK", 1: "EAGLE_ATTN_DEV_BAD_CU_SEQLENS",
              2: "EAGLE_ATTN_DEV_DOC_TOO_LONG", 3: "EAGLE_ATTN_DEV_POS_OUTSIDE",
              4: "EAGLE_ATTN_DEV_TIMEOUT", 5: "EAGLE_ATTN_DEV_BAD_TILE",
              6: "EAGLE_ATTN_DEV_SMEM_ALIGN"}

F32, BF16 = 0, 1
GRAD_STORE, GRAD_ACCUMULATE_F32 = 0, 1
IMPL = {"auto": 0, "tensor_core": 1, "generic": 2}

# Every function declared in include/eagleattn.h.
EXPORTS = (
    "eagle_attn_abi_version", "eagle_attn_params_init", "eagle_attn_fwd",
    "eagle_attn_bwd_workspace_size", "eagle_attn_bwd", "attn_merge_out_lse", "attn_merge_diag",
    "attn_finalize", "eagle_attn_get_status", "eagle_attn_clear_status", "eagle_attn_strerror",
    "eagle_attn_launch_count", "eagle_attn_bwd_noalloc", "eagle_attn_selftest_wait_timeout",
)


class Params(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32),
        ("abi_version", ctypes.c_uint32),
        ("dtype", ctypes.c_int32),
        ("out_dtype", ctypes.c_int32),
        ("impl", ctypes.c_int32),
        ("B", ctypes.c_int32), ("Tq", ctypes.c_int32), ("Tk", ctypes.c_int32),
        ("H", ctypes.c_int32), ("D", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("deterministic", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("q_pos_offset", ctypes.c_int64),
        ("k_pos_offset", ctypes.c_int64),
        ("cu_seqlens", ctypes.c_void_p),
        ("num_docs", ctypes.c_int32),
        ("max_seqlen", ctypes.c_int32),
        ("q_stride_b", ctypes.c_int64), ("q_stride_t", ctypes.c_int64),
        ("kv_stride_b", ctypes.c_int64), ("kv_stride_blk", ctypes.c_int64),
        ("kv_stride_t", ctypes.c_int64),
        ("q", ctypes.c_void_p), ("cache_k", ctypes.c_void_p), ("cache_v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("grad_out", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p),
        ("dv", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("prof_start", ctypes.c_void_p), ("prof_stop", ctypes.c_void_p),
        ("grad_mode", ctypes.c_int32),
        ("q_tiles", ctypes.c_void_p), ("num_q_tiles", ctypes.c_int32),
        ("q_tile_rows", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libeagleattn.so is not built (run `python -m online_softmax_merge_eagle_b200.build`); "
            "there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.eagle_attn_abi_version.restype = i32
    lib.eagle_attn_abi_version.argtypes = []
    lib.eagle_attn_params_init.restype = None
    lib.eagle_attn_params_init.argtypes = [P]
    lib.eagle_attn_fwd.restype = i32
    lib.eagle_attn_fwd.argtypes = [P, vp]
    lib.eagle_attn_bwd_workspace_size.restype = sz
    lib.eagle_attn_bwd_workspace_size.argtypes = [P]
    lib.eagle_attn_bwd.restype = i32
    lib.eagle_attn_bwd.argtypes = [P, vp]
    lib.eagle_attn_bwd_noalloc.restype = i32
    lib.eagle_attn_bwd_noalloc.argtypes = [P, vp]
    lib.attn_merge_out_lse.restype = i32
    lib.attn_merge_out_lse.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, vp]
    lib.attn_merge_diag.restype = i32
    lib.attn_merge_diag.argtypes = [P, vp]
    lib.attn_finalize.restype = i32
    lib.attn_finalize.argtypes = [vp, vp, i32, sz, vp]
    lib.eagle_attn_get_status.restype = i32
    lib.eagle_attn_get_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
    lib.eagle_attn_clear_status.restype = i32
    lib.eagle_attn_clear_status.argtypes = []
    lib.eagle_attn_launch_count.restype = ctypes.c_uint64
    lib.eagle_attn_launch_count.argtypes = []
    lib.eagle_attn_selftest_wait_timeout.restype = i32
    lib.eagle_attn_selftest_wait_timeout.argtypes = [ctypes.c_int64, vp]
    lib.eagle_attn_strerror.restype = ctypes.c_char_p
    lib.eagle_attn_strerror.argtypes = [i32]
    if lib.eagle_attn_abi_version() != ABI_VERSION:
        raise RuntimeError("libeagleattn ABI version mismatch")
    _lib = lib
    return lib
