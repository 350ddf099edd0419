"""ctypes binding of libwise.so (the C ABI declared in include/wise.h).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of the library.  Importing this module without a built library
raises ImportError; there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libwise.so")

WISE_OK = 0
WISE_ERR_ARG = -1
WISE_ERR_SHAPE = -2
WISE_ERR_ALIGN = -3
WISE_ERR_CAPACITY = -4
WISE_ERR_CUDA = -5
WISE_ERR_WORKSPACE = -6

WISE_STATUS_TIMEOUT = 0x1
WISE_STATUS_BAD_SCHEDULE = 0x2

ERROR_NAMES = {
    WISE_ERR_ARG: "WISE_ERR_ARG", WISE_ERR_SHAPE: "WISE_ERR_SHAPE",
    WISE_ERR_ALIGN: "WISE_ERR_ALIGN", WISE_ERR_CAPACITY: "WISE_ERR_CAPACITY",
    WISE_ERR_CUDA: "WISE_ERR_CUDA", WISE_ERR_WORKSPACE: "WISE_ERR_WORKSPACE",
}


class WiseShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("seqlen", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("scale", ctypes.c_float), ("kv_heads", ctypes.c_int32)]


class WiseError(RuntimeError):
    def __init__(self, code: int, func: str, msg: str):
        super().__init__(f"{func}: {ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


_vp = ctypes.c_void_p
_SIGNATURES = {
    "wise_full_attn_mass": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                           WiseShape, _vp]),
    "wise_mass_workspace_bytes": (ctypes.c_size_t, [WiseShape]),
    "wise_window_step": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                                        _vp, ctypes.c_size_t, WiseShape, _vp]),
    "wise_select_union": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_float, WiseShape, _vp]),
    "wise_select_union_blocks": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_float, ctypes.c_int32,
                                                WiseShape, _vp]),
    "wise_block_mass_b16": (ctypes.c_int, [_vp, _vp, _vp, _vp, WiseShape, _vp]),
    "wise_full_attn_mass_b16": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                               ctypes.c_size_t, WiseShape, _vp]),
    "wise_mass_b16_workspace_bytes": (ctypes.c_size_t, [WiseShape]),
    "wise_select_union_b16": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_float, WiseShape, _vp]),
    "wise_schedule_b16_workspace_bytes": (ctypes.c_size_t, [WiseShape]),
    "wise_build_schedule_b16": (ctypes.c_int, [_vp, _vp, _vp, _vp, ctypes.c_int64,
                                               ctypes.POINTER(ctypes.c_int64), _vp,
                                               ctypes.c_size_t, WiseShape, _vp]),
    "wise_sparse_attn_b16": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int64,
                                            _vp, WiseShape, _vp]),
    "wise_select_size_matched": (ctypes.c_int, [_vp, _vp, _vp, WiseShape, _vp]),
    "wise_select_mass_matched": (ctypes.c_int, [_vp, _vp, _vp, WiseShape, _vp]),
    "wise_support_mass": (ctypes.c_int, [_vp, _vp, _vp, WiseShape, _vp]),
    "wise_schedule_workspace_bytes": (ctypes.c_size_t, [WiseShape]),
    "wise_schedule_max_nnz": (ctypes.c_int64, [WiseShape]),
    "wise_build_schedule": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int64,
                                           ctypes.POINTER(ctypes.c_int64), _vp, ctypes.c_size_t,
                                           WiseShape, _vp]),
    "wise_build_schedule_static": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int64,
                                                  ctypes.POINTER(ctypes.c_int64), WiseShape, _vp]),
    "wise_sparse_attn": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int64, _vp,
                                        WiseShape, _vp]),
    "wise_diag_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, _vp]),
    "wise_device_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]),
    "wise_last_error": (ctypes.c_char_p, []),
    "wise_version": (ctypes.c_char_p, []),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python recurrent_depth_lm_b200/build.py` "
            "(or __graft_entry__.build()) first. There is no non-CUDA fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def last_error() -> str:
    return lib.wise_last_error().decode()


def check(code: int, func: str) -> None:
    if code != WISE_OK:
        raise WiseError(code, func, last_error())


def version() -> str:
    return lib.wise_version().decode()
