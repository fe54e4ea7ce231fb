"""ctypes declarations of liblmh.so (include/lmh.h). Loading fails loudly if it is not built."""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblmh.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "lmh.h")

c_int64, c_uint32, c_int, c_size_t, c_void_p = (ctypes.c_int64, ctypes.c_uint32, ctypes.c_int,
                                                ctypes.c_size_t, ctypes.c_void_p)

LMH_OK = 0
STATUS_NAMES = {0: "LMH_OK", 1: "LMH_ERR_INVALID_ARG", 2: "LMH_ERR_UNSUPPORTED_DEVICE",
                3: "LMH_ERR_WORKSPACE_TOO_SMALL", 4: "LMH_ERR_ALIGNMENT", 5: "LMH_ERR_CUDA",
                6: "LMH_ERR_SCRATCH_LIMIT"}

IGNORE_INDEX = -100
DEVERR_LABEL_RANGE, DEVERR_TIMEOUT, DEVERR_NONFINITE, DEVERR_TEMPERATURE = 0x1, 0x2, 0x4, 0x8
F_MEAN, F_FUSED_BWD, F_DW_ACC_GIVEN, F_SUPPORT_RENORM, F_GRAD_SCALAR = 0x1, 0x2, 0x4, 0x8, 0x10
F_DW_ACC_STORE = 0x20
ENTRY_LOSS_FWD, ENTRY_LOSS_BWD, ENTRY_LOGPROB, ENTRY_SUPPORT_LOGPROB, ENTRY_SUPPORT_KL = range(5)
ENTRY_VP_PARTIALS, ENTRY_VP_COMBINE, ENTRY_VP_BWD, ENTRY_LOSS_FWD_BWD = 5, 6, 7, 8
ENTRY_VP_SUPPORT_PARTIALS, ENTRY_VP_SUPPORT_COMBINE, ENTRY_VP_SUPPORT_BWD = 9, 10, 11
BWD_CE, BWD_LOGPROB, BWD_SUPPORT_LOGPROB, BWD_SUPPORT_KL = range(4)
MAX_K = 1024


class lmh_shape(ctypes.Structure):
    _fields_ = [("N", c_int64), ("d", c_int64), ("V", c_int64), ("K", c_int64),
                ("chunk_rows", c_int64), ("flags", c_uint32), ("temperature", ctypes.c_float),
                ("row_temperature", c_void_p)]


class lmh_vp_dest(ctypes.Structure):
    _fields_ = [("recv", c_void_p), ("R", ctypes.c_int32), ("rank", ctypes.c_int32)]


_P = c_void_p
_SIGS = {
    "lmh_workspace_size": (c_size_t, [ctypes.POINTER(lmh_shape), c_int]),
    "lmh_dh_plan": (c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _P, _P]),
    "lmh_loss_fwd": (c_int, [ctypes.POINTER(lmh_shape)] + [_P] * 14 + [c_size_t, _P]),
    "lmh_loss_bwd": (c_int, [ctypes.POINTER(lmh_shape), c_int] + [_P] * 10 + [c_size_t, _P]),
    "lmh_loss_fwd_bwd": (c_int, [ctypes.POINTER(lmh_shape), c_int] + [_P] * 15 + [c_size_t, _P]),
    "lmh_logprob": (c_int, [ctypes.POINTER(lmh_shape)] + [_P] * 6 + [c_size_t, _P]),
    "lmh_support_logprob": (c_int, [ctypes.POINTER(lmh_shape)] + [_P] * 6 + [c_size_t, _P]),
    "lmh_support_kl": (c_int, [ctypes.POINTER(lmh_shape)] + [_P] * 9 + [c_size_t, _P]),
    "lmh_vp_partials": (c_int, [ctypes.POINTER(lmh_shape), c_int64, c_int64] + [_P] * 5
                        + [c_size_t, _P]),
    "lmh_vp_combine": (c_int, [ctypes.POINTER(lmh_shape), c_int] + [_P] * 10 + [c_size_t, _P]),
    "lmh_vp_loss_bwd": (c_int, [ctypes.POINTER(lmh_shape), c_int, c_int64, c_int64] + [_P] * 8
                        + [ctypes.POINTER(lmh_vp_dest), _P, c_size_t, _P]),
    "lmh_vp_fused_bwd": (c_int, [ctypes.POINTER(lmh_shape), c_int64, c_int64] + [_P] * 8
                         + [ctypes.POINTER(lmh_vp_dest), _P, c_size_t, _P]),
    "lmh_vp_reduce_rows_to": (c_int, [c_int, c_int64, c_int64, _P, _P, c_int, c_int64, _P]),
    "lmh_vp_support_partials": (c_int, [ctypes.POINTER(lmh_shape), c_int64, c_int64] + [_P] * 5
                                + [c_size_t, _P]),
    "lmh_vp_support_combine": (c_int, [ctypes.POINTER(lmh_shape), c_int] + [_P] * 8
                               + [c_size_t, _P]),
    "lmh_vp_support_bwd": (c_int, [ctypes.POINTER(lmh_shape), c_int, c_int64, c_int64] + [_P] * 9
                           + [ctypes.POINTER(lmh_vp_dest), _P, c_size_t, _P]),
    "lmh_vp_reduce_rows": (c_int, [c_int, c_int64, c_int64, _P, _P, _P]),
    "lmh_support_kl_fwd_bwd": (c_int, [ctypes.POINTER(lmh_shape)] + [_P] * 12 + [c_size_t, _P]),
    "lmh_support_fwd_bwd": (c_int, [ctypes.POINTER(lmh_shape), c_int] + [_P] * 13
                            + [c_size_t, _P]),
    "lmh_scale_bf16": (c_int, [_P, c_int64, _P, _P]),
    "lmh_count_valid": (c_int, [c_int64, c_int64, _P, _P, _P]),
    "lmh_dp_loss_fwd_bwd": (c_int, [ctypes.POINTER(lmh_shape), c_int] + [_P] * 11
                            + [ctypes.POINTER(lmh_vp_dest), _P, c_size_t, _P]),
    "lmh_reduce_ranks_f32": (c_int, [c_int, c_int64, _P, _P, _P]),
    "lmh_read_errors": (c_int, [_P, ctypes.POINTER(c_uint32), _P]),
    "lmh_logprob_noalloc": (c_int, [ctypes.POINTER(lmh_shape)] + [_P] * 6),
    "lmh_peer_barrier": (c_int, [_P, _P, ctypes.c_int32, ctypes.c_int32, c_uint32, c_uint32, _P]),
    "lmh_selftest_wait_timeout": (c_int, [_P, c_uint32, _P]),
    "lmh_profile_enable": (c_int, [c_int]),
    "lmh_profile_read": (c_int, [c_int, ctypes.POINTER(ctypes.c_int32),
                                 ctypes.POINTER(ctypes.c_float)]),
    "lmh_kernel_name": (ctypes.c_char_p, [c_int]),
}


def header_symbols(path: str = HEADER):
    """Names of the functions include/lmh.h declares."""
    src = open(path).read()
    return re.findall(r"^LMH_API\s+[\w\s\*]*?\b(lmh_\w+)\s*\(", src, flags=re.M)


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        hint = "run `python lm_head_cross_tcgen05_b200/build.py` (this package has no fallback path)"
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; {hint}")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            try:
                f = getattr(L, name)
            except AttributeError:
                raise ImportError(f"{LIB_PATH} lacks {name}: it is older than its sources; {hint}")
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib
