"""ctypes binding of libquip (include/quip.h).  Argument marshalling only:
every step of the computation runs in the library's CUDA kernels."""
from __future__ import annotations

import ctypes
import os
from ctypes import c_char_p, c_float, c_int, c_int64, c_size_t, c_uint64, c_void_p, POINTER

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libquip.so")

QUIP_OK, QUIP_ERR_ARG, QUIP_ERR_SHAPE, QUIP_ERR_UNSUPPORTED = 0, 1, 2, 3
QUIP_ERR_NOT_PD, QUIP_ERR_NONFINITE, QUIP_ERR_CUDA, QUIP_ERR_TIMEOUT, QUIP_ERR_WORKSPACE = 4, 5, 6, 7, 8
QUIP_F32, QUIP_BF16, QUIP_U8 = 0, 1, 2
QUIP_T_IDENTITY, QUIP_T_HADAMARD, QUIP_T_KRONECKER = 0, 1, 2
QUIP_T_PERMUTE = 0x100
QUIP_OP_INCOHERENCE_FORWARD, QUIP_OP_INCOHERENCE_INVERSE, QUIP_OP_LDL, QUIP_OP_LDLQ = 0, 1, 2, 3
QUIP_OP_GREEDY, QUIP_OP_QMATVEC = 4, 5

# name -> (restype, argtypes); the list of every symbol include/quip.h declares
SIGNATURES = {
    "quip_status_string": (c_char_p, [c_int]),
    "quip_version": (c_char_p, []),
    "quip_kernel_launches": (c_uint64, []),
    "quip_transform_create": (c_int, [c_uint64, c_int64, c_int64, c_int, c_int64, c_int64, c_int,
                                      c_int64, c_int64, c_void_p, POINTER(c_void_p)]),
    "quip_transform_destroy": (c_int, [c_void_p]),
    "quip_transform_draw": (c_int, [c_void_p, c_uint64, c_void_p]),
    "quip_transform_info": (c_int, [c_void_p, c_int, POINTER(c_int), POINTER(c_int64),
                                    POINTER(c_int64), POINTER(c_void_p), POINTER(c_void_p),
                                    POINTER(c_void_p)]),
    "quip_transform_permutation": (c_int, [c_void_p, c_int, POINTER(c_void_p)]),
    "quip_hessian_accumulate": (c_int, [c_void_p, c_int, c_int64, c_int64, c_int64, c_void_p, c_int,
                                        c_void_p]),
    "quip_hessian_finalize": (c_int, [c_void_p, c_int64, c_int64, c_float, c_void_p]),
    "quip_incoherence_forward": (c_int, [c_void_p, c_void_p, c_int, c_int64, c_void_p, c_void_p,
                                         c_void_p, c_size_t, c_void_p]),
    "quip_incoherence_inverse": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "quip_ldl": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_size_t, c_void_p]),
    "quip_ldlq_quantize": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int, c_int64,
                                   c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "quip_ldlq_quantize_static": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int,
                                          c_int64, c_void_p, c_void_p, c_void_p, c_void_p]),
    "quip_nearest_quantize": (c_int, [c_void_p, c_int64, c_int64, c_int, c_void_p, c_void_p, c_void_p,
                                      c_void_p]),
    "quip_diag_order": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p]),
    "quip_permute": (c_int, [c_void_p, c_int, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                             c_int64, c_void_p]),
    "quip_greedy_refine": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int, c_void_p,
                                   c_void_p, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "quip_packed_words": (c_int64, [c_int64, c_int]),
    "quip_pack_codes": (c_int, [c_void_p, c_int64, c_int64, c_int, c_void_p, c_int64, c_void_p]),
    "quip_qmatvec": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_int, c_void_p, c_int,
                             c_int64, c_int64, c_void_p, c_int64, c_void_p, c_size_t, c_void_p]),
    "quip_dequantize": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_void_p]),
    "quip_workspace_size": (c_int, [c_int, c_void_p, c_int64, c_int64, c_int64, POINTER(c_size_t)]),
    "quip_quantize_layer": (c_int, [c_void_p, c_uint64, c_void_p, c_int, c_int64, c_void_p, c_int, c_int64,
                                    c_int64, c_int, c_int64, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_size_t, c_void_p]),
    "quip_quantize_layer_host": (c_int, [c_void_p, c_uint64, c_void_p, c_int, c_int64, c_void_p, c_int,
                                         c_int64, c_int64, c_int, c_int64, c_float, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "quip_layer_workspace_size": (c_int, [c_void_p, c_int64, c_int, c_int, c_int64, c_int, POINTER(c_size_t)]),
    "quip_sync_status": (c_int, [c_void_p]),
    "quip_timing_begin": (c_int, []),
    "quip_timing_end": (c_int, [POINTER(c_char_p), POINTER(c_uint64), POINTER(ctypes.c_double), c_int,
                                POINTER(c_int)]),
    "quip_timing_trace": (c_int, [POINTER(c_char_p), POINTER(ctypes.c_double), POINTER(ctypes.c_double),
                                  POINTER(c_int), c_int, POINTER(c_int)]),
}

_lib = None


class QuipError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libquip.so; raises if it was not built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libquip.so not found at {path}: build it with "
                           "`python post_weight_quantization_09_b200/build.py`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().quip_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != QUIP_OK:
        raise QuipError(status, where)
