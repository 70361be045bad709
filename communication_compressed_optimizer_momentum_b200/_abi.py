"""ctypes declarations of the C ABI in ``include/onebit_adam.h``.

Loading fails loudly: if ``libonebit_adam.so`` has not been built there is no fallback of any
kind; every computation of the method runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libonebit_adam.so")

P = ctypes.c_void_p
I32, I64, U32P, U64P = ctypes.c_int32, ctypes.c_int64, ctypes.POINTER(ctypes.c_uint32), \
    ctypes.POINTER(ctypes.c_uint64)
F32 = ctypes.c_float
INT = ctypes.c_int

# name -> (restype, argtypes); mirrors include/onebit_adam.h
SIGNATURES = {
    "onebit_adam_init": (INT, [ctypes.POINTER(P), I64, I32, I64, F32, F32, F32]),
    "onebit_adam_workspace_bytes": (INT, [P, I32, U64P]),
    "onebit_adam_bind": (INT, [P, P, ctypes.c_uint64, I32, P]),
    "onebit_adam_warmup_step": (INT, [P, P, P, F32, P]),
    "onebit_adam_freeze_variance": (INT, [P, P]),
    "onebit_adam_set_bias_correction": (INT, [P, I32]),
    "onebit_adam_compressed_step": (INT, [P, P, P, F32, P]),
    "onebit_adam_compressed_step_host": (INT, [P, P, P, P, P, F32, P]),
    "onebit_adam_host_wait": (INT, [P, P]),
    "onebit_adam_get_state": (INT, [P, I32, P, P]),
    "onebit_adam_get_chunk_state": (INT, [P, I32, I64, P, P]),
    "onebit_adam_set_state": (INT, [P, I32, P, P]),
    "onebit_adam_state_bytes": (INT, [P, I32, U64P]),
    "onebit_adam_status": (INT, [P, P, U32P]),
    "onebit_adam_info": (INT, [P, ctypes.POINTER(I64)]),
    "onebit_adam_timing": (INT, [P, I32]),
    "onebit_adam_timing_read": (INT, [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I32)]),
    "onebit_adam_timing_steps": (INT, [P, ctypes.POINTER(ctypes.c_double), I32,
                                       ctypes.POINTER(I32)]),
    "onebit_adam_destroy": (None, [P]),
    "onebit_pack": (INT, [P, I64, P, P]),
    "onebit_unpack": (INT, [P, P, I64, I64, P, P]),
    "onebit_compress_static": (INT, [P, I64, I64, P, P, P]),
    "onebit_selftest_bounded_wait": (INT, [I32, P, P]),
    "onebit_server_layout": (INT, [I64, I32, I64, ctypes.POINTER(I64)]),
    "onebit_dp_chunk_range": (INT, [I64, I32, I32, ctypes.POINTER(I64), ctypes.POINTER(I64)]),
    "onebit_dp_init": (INT, [ctypes.POINTER(P), I64, I32, I64, F32, F32, F32, I32, I32]),
    "onebit_dp_info": (INT, [P, ctypes.POINTER(I64)]),
    "onebit_dp_exchange": (INT, [P, ctypes.POINTER(P), U64P]),
    "onebit_dp_ipc_handle": (INT, [P, P]),
    "onebit_dp_open_peer": (INT, [P, I32, P]),
    "onebit_dp_set_peer": (INT, [P, I32, P]),
    "onebit_dp_connect": (INT, [P, P]),
    "onebit_dp_set_timeout": (INT, [P, ctypes.c_uint64]),
    "onebit_dp_warmup_phase": (INT, [P, I32, P, P, F32, P]),
    "onebit_dp_compressed_phase": (INT, [P, I32, P, P, F32, P]),
    "onebit01_init": (INT, [ctypes.POINTER(P), I64, I32, I64, F32, F32, F32, I32, I32]),
    "onebit01_step": (INT, [P, P, P, F32, P]),
    "onebit01_info": (INT, [P, ctypes.POINTER(I64)]),
    "onebit01_get_worker_state": (INT, [P, I32, I64, P, P]),
    "onebit01_local_model": (INT, [P, I32, P, P, P]),
    "onebit01_set_worker_state": (INT, [P, I32, P, P]),
    "onebit01_get_schedule": (INT, [P, ctypes.POINTER(I64), ctypes.POINTER(F32)]),
    "onebit01_set_schedule": (INT, [P, ctypes.POINTER(I64), ctypes.POINTER(F32)]),
    "onebit01_dp_init": (INT, [ctypes.POINTER(P), I64, I32, I64, F32, F32, F32, I32, I32, I32,
                               I32]),
    "onebit01_dp_phase": (INT, [P, I32, P, P, F32, P]),
    "onebit_strerror": (ctypes.c_char_p, [I32]),
    "onebit_last_error": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libonebit_adam.so is not built (expected at %s); run "
                "`python -m communication_compressed_optimizer_momentum_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib
