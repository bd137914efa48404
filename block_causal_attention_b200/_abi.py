"""ctypes binding of libbca.so (include/bca.h).  Argument marshalling only: every
step of the computation runs in the library's CUDA kernels.  Loading fails loudly
when the library has not been built."""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbca.so")

BCA_OK = 0
BCA_ERR_INVALID_ARGUMENT = -1
BCA_ERR_BAD_SLICE = -2
BCA_ERR_UNSUPPORTED = -3
BCA_ERR_MISALIGNED = -4
BCA_ERR_CUDA = -5
BCA_ERR_DEVICE_TIMEOUT = -6
BCA_ERR_HOST_ONLY_PLAN = -7
BCA_ERR_NO_MEMORY = -8
BCA_ERR_TOO_LARGE = -9
BCA_STATIC_WORKSPACE_BYTES = 16 << 20

BCA_SLICE_FULL = 0
BCA_SLICE_CAUSAL = 1
BCA_O_FP32 = 0x1
BCA_PLAN_HOST_ONLY = 0x2
BCA_TEST_FORCE_TIMEOUT = 0x4
BCA_FWD_FP8_E4M3 = 0x8
BCA_NO_PROLOGUE = 0x10
BCA_DQ_DETERMINISTIC = 0x20
BCA_CACHE_K_FP16 = 0x40
BCA_PASS_FWD = 0
BCA_PASS_BWD = 1

# every symbol include/bca.h declares
EXPORTS = ("bca_plan_create", "bca_plan_destroy", "bca_plan_get_info", "bca_plan_expand_rows",
           "bca_plan_expand_cols",
           "bca_plan_update_positions", "bca_workspace_bytes", "bca_fwd", "bca_fwd_static_workspace", "bca_bwd",
           "bca_bwd_ex", "bca_attn_merge", "bca_k_prologue", "bca_k_prologue_bwd",
           "bca_profile_enable",
           "bca_profile_read", "bca_status", "bca_error_string")
BCA_KERNEL_KV_IMAGE = 0
BCA_KERNEL_FWD = 1
KERNEL_NAMES = {0: "kv_image_kernel", 1: "fwd_kernel", 2: "bwd_prep_kernel", 3: "bwd_kv_image_kernel",
                4: "bwd_kernel", 5: "bwd_dq_kernel", 6: "bwd_dq_pass_kernel"}


class bca_slice(ctypes.Structure):
    _fields_ = [("q_begin", ctypes.c_int64), ("q_end", ctypes.c_int64), ("k_begin", ctypes.c_int64),
                ("k_end", ctypes.c_int64), ("type", ctypes.c_int64)]


class bca_video(ctypes.Structure):
    _fields_ = [("num_chunks", ctypes.c_int32), ("frames", ctypes.c_int32), ("height", ctypes.c_int32),
                ("width", ctypes.c_int32), ("t0", ctypes.c_int32)]


class bca_problem(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("num_videos", ctypes.c_int32),
                ("videos", ctypes.c_void_p), ("num_cache_keys", ctypes.c_int64),
                ("num_slices", ctypes.c_int32), ("slices", ctypes.c_void_p),
                ("rope_base", ctypes.c_float * 3), ("norm_eps", ctypes.c_float),
                ("flags", ctypes.c_uint32)]


class bca_plan_info(ctypes.Structure):
    _fields_ = [("num_q", ctypes.c_int64), ("num_k", ctypes.c_int64), ("num_cache", ctypes.c_int64),
                ("num_q_tiles", ctypes.c_int64), ("num_k_tiles", ctypes.c_int64),
                ("num_runs", ctypes.c_int64), ("num_full_tiles", ctypes.c_int64),
                ("num_partial_tiles", ctypes.c_int64), ("num_items", ctypes.c_int64),
                ("visible_pairs", ctypes.c_int64), ("head_dim_padded", ctypes.c_int32),
                ("tile_q", ctypes.c_int32), ("tile_k", ctypes.c_int32)]


_lib = None


class BcaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} ({code})")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libbca.so is not built ({LIB_PATH}); run "
                              "`python -m block_causal_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.bca_plan_create.argtypes = [ctypes.POINTER(bca_problem), ctypes.POINTER(vp)]
        L.bca_plan_create.restype = i32
        L.bca_plan_destroy.argtypes = [vp]
        L.bca_plan_destroy.restype = None
        L.bca_plan_get_info.argtypes = [vp, ctypes.POINTER(bca_plan_info)]
        L.bca_plan_get_info.restype = i32
        L.bca_plan_expand_rows.argtypes = [vp, i64, i64, vp]
        L.bca_plan_expand_rows.restype = i32
        L.bca_plan_expand_cols.argtypes = [vp, i64, i64, vp]
        L.bca_plan_expand_cols.restype = i32
        L.bca_workspace_bytes.argtypes = [vp, i32]
        L.bca_workspace_bytes.restype = ctypes.c_size_t
        L.bca_fwd.argtypes = [vp] * 12
        L.bca_fwd.restype = i32
        L.bca_plan_update_positions.argtypes = [vp, vp, i32, vp]
        L.bca_plan_update_positions.restype = i32
        L.bca_attn_merge.argtypes = [vp] * 8
        L.bca_attn_merge.restype = i32
        L.bca_k_prologue.argtypes = [vp] * 5
        L.bca_k_prologue.restype = i32
        L.bca_k_prologue_bwd.argtypes = [vp, vp, vp, vp, vp, i32, vp]
        L.bca_k_prologue_bwd.restype = i32
        L.bca_bwd.argtypes = [vp] * 18
        L.bca_bwd.restype = i32
        L.bca_bwd_ex.argtypes = [vp] * 19 + [i32, vp, vp]
        L.bca_bwd_ex.restype = i32
        L.bca_fwd_static_workspace.argtypes = [vp] * 11
        L.bca_fwd_static_workspace.restype = i32
        L.bca_profile_enable.argtypes = [vp, i32]
        L.bca_profile_enable.restype = i32
        L.bca_profile_read.argtypes = [vp, i32, ctypes.POINTER(i64), ctypes.POINTER(ctypes.c_double)]
        L.bca_profile_read.restype = i32
        L.bca_status.argtypes = [vp, vp]
        L.bca_status.restype = i32
        L.bca_error_string.argtypes = [i32]
        L.bca_error_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().bca_error_string(int(code)).decode()


def check(code: int, where: str) -> None:
    if code != BCA_OK:
        raise BcaError(code, where)


def make_problem(hq, hkv, d, videos, num_cache_keys, slices, rope_base=(1e4, 1e4, 1e4),
                 eps=1e-6, flags=0):
    """Build a bca_problem; returns (problem, keepalive) - keep both alive while the
    problem is used."""
    vid = np.ascontiguousarray(np.asarray(videos, dtype=np.int32).reshape(-1, 5))
    p = bca_problem()
    p.num_q_heads, p.num_kv_heads, p.head_dim = int(hq), int(hkv), int(d)
    p.num_videos = len(vid)
    p.videos = vid.ctypes.data if len(vid) else None
    p.num_cache_keys = int(num_cache_keys)
    keep = [vid]
    if slices is None:
        p.num_slices, p.slices = 0, None
    else:
        sl = np.ascontiguousarray(np.asarray(slices, dtype=np.int64).reshape(-1, 5))
        # an explicit empty list means "no visible pair" (NULL means the default
        # block-causal mask), so always pass a non-NULL pointer here
        buf = sl if len(sl) else np.zeros((1, 5), np.int64)
        keep.append(buf)
        p.num_slices = len(sl)
        p.slices = buf.ctypes.data
    p.rope_base[:] = [float(x) for x in rope_base]
    p.norm_eps = float(eps)
    p.flags = int(flags)
    return p, keep
