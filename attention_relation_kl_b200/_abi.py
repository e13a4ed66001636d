"""ctypes declarations of librelkl.so (include/relkl.h).  Marshalling only."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librelkl.so")

RELKL_OK = 0
RELKL_ERR_INVALID = 1
RELKL_ERR_UNSUPPORTED = 2
RELKL_ERR_CUDA = 3
RELKL_ERR_WORKSPACE = 4
RELKL_ERR_TIMEOUT = 5
RELKL_BF16 = 0
RELKL_FP32 = 1

# Every symbol include/relkl.h declares.
EXPORTS = ("relkl_workspace_bytes", "relkl_workspace_init", "relkl_fwd", "relkl_bwd",
           "relkl_fwd_qkv", "relkl_bwd_qkv", "relkl_get_device_error",
           "relkl_set_wait_timeout_ns", "relkl_status_string", "relkl_last_cuda_error",
           "relkl_path_for", "relkl_fwd_noalloc", "relkl_rope_bwd", "relkl_weight_grad",
           "relkl_cast_bf16", "relkl_bwd_kernel_for",
           "relkl_fwd_qkv_part", "relkl_bwd_qkv_part", "relkl_check_schedule")


class relkl_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("stride", ctypes.c_int64 * 4), ("dtype", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("scale", ctypes.c_float),
                ("reserved", ctypes.c_int32), ("lengths", ctypes.c_void_p),
                ("cu_seqlens", ctypes.c_void_p), ("n_seq", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int32)]


class relkl_rope(ctypes.Structure):
    _fields_ = [("base", ctypes.c_double), ("pos_scale", ctypes.c_double),
                ("pos_offset", ctypes.c_double), ("apply", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_vp = ctypes.c_void_p
_fp = ctypes.POINTER(ctypes.c_float)
_PV = ctypes.POINTER(ctypes.c_void_p)


def _declare(lib):
    lib.relkl_workspace_bytes.restype = ctypes.c_size_t
    lib.relkl_workspace_bytes.argtypes = []
    lib.relkl_workspace_init.restype = ctypes.c_int
    lib.relkl_workspace_init.argtypes = [_vp, ctypes.c_size_t, _vp]
    lib.relkl_fwd.restype = ctypes.c_int
    lib.relkl_fwd.argtypes = [ctypes.POINTER(relkl_desc), _vp, _vp, _vp, _vp, _vp,
                              ctypes.c_size_t, _vp]
    lib.relkl_bwd.restype = ctypes.c_int
    lib.relkl_bwd.argtypes = [ctypes.POINTER(relkl_desc), _vp, _vp, _vp, _vp, _vp, _vp,
                              ctypes.c_size_t, _vp]
    lib.relkl_fwd_qkv.restype = ctypes.c_int
    lib.relkl_fwd_qkv.argtypes = [ctypes.c_int32, ctypes.POINTER(relkl_desc), _PV, _PV, _PV, _PV,
                                  _vp, ctypes.c_size_t, _vp]
    lib.relkl_bwd_qkv.restype = ctypes.c_int
    lib.relkl_bwd_qkv.argtypes = [ctypes.c_int32, ctypes.POINTER(relkl_desc), _PV, _PV, _PV, _PV,
                                  _PV, _vp, ctypes.c_size_t, _vp]
    lib.relkl_fwd_qkv_part.restype = ctypes.c_int
    lib.relkl_fwd_qkv_part.argtypes = [ctypes.c_int32, ctypes.POINTER(relkl_desc), _PV, _PV, _PV,
                                       _PV, ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_size_t,
                                       _vp]
    lib.relkl_bwd_qkv_part.restype = ctypes.c_int
    lib.relkl_bwd_qkv_part.argtypes = [ctypes.c_int32, ctypes.POINTER(relkl_desc), _PV, _PV, _PV,
                                       _PV, _PV, ctypes.c_int32, ctypes.c_int32, _vp,
                                       ctypes.c_size_t, _vp]
    lib.relkl_check_schedule.restype = ctypes.c_int
    lib.relkl_check_schedule.argtypes = [ctypes.c_int32, ctypes.POINTER(relkl_desc), ctypes.c_int32,
                                         ctypes.c_int32, _PV, _PV, ctypes.c_char_p, ctypes.c_size_t]
    lib.relkl_get_device_error.restype = ctypes.c_int
    lib.relkl_get_device_error.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.relkl_set_wait_timeout_ns.restype = ctypes.c_uint64
    lib.relkl_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.relkl_status_string.restype = ctypes.c_char_p
    lib.relkl_status_string.argtypes = [ctypes.c_int]
    lib.relkl_last_cuda_error.restype = ctypes.c_int32
    lib.relkl_last_cuda_error.argtypes = []
    lib.relkl_path_for.restype = ctypes.c_int32
    lib.relkl_path_for.argtypes = [ctypes.POINTER(relkl_desc)]
    lib.relkl_fwd_noalloc.restype = ctypes.c_int
    lib.relkl_fwd_noalloc.argtypes = [ctypes.POINTER(relkl_desc), _vp, _vp, _vp, _vp, _vp]
    i32 = ctypes.c_int32
    lib.relkl_bwd_kernel_for.restype = ctypes.c_int32
    lib.relkl_bwd_kernel_for.argtypes = [ctypes.c_int32, ctypes.POINTER(relkl_desc), ctypes.c_int32]
    lib.relkl_cast_bf16.restype = ctypes.c_int
    lib.relkl_cast_bf16.argtypes = [_vp, _vp, ctypes.c_int64, _vp]
    lib.relkl_rope_bwd.restype = ctypes.c_int
    lib.relkl_rope_bwd.argtypes = [i32, i32, i32, i32, _vp, ctypes.POINTER(relkl_rope), i32, _vp, _vp]
    lib.relkl_weight_grad.restype = ctypes.c_int
    lib.relkl_weight_grad.argtypes = [ctypes.c_int64, i32, i32, _vp, _vp, _vp, _vp,
                                      ctypes.c_size_t, _vp]
    return lib


_LIB = None


def lib():
    """The loaded library.  Raises if the CUDA extension has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"librelkl.so is missing ({LIB_PATH}); build it with "
                              "`python -m attention_relation_kl_b200.build`")
        _LIB = _declare(ctypes.CDLL(LIB_PATH))
    return _LIB


class RelklError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = lib().relkl_status_string(code).decode()
        if code == RELKL_ERR_CUDA:
            msg += f" (CUDA status {lib().relkl_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")
        self.code = code


def check(code: int, where: str) -> None:
    if code != RELKL_OK:
        raise RelklError(code, where)
