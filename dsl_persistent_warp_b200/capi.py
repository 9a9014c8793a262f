"""ctypes binding of the C ABI in include/gemm_bf16.h, under the same names.

Argument marshalling only: each function here forwards to the symbol of the same name in
libgemm_bf16.so.  The library must have been built (``dsl_persistent_warp_b200._build``);
importing this module without it raises, and there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

from ._build import LIB_PATH

GEMM_OK = 0
GEMM_ERR_INVALID_ARG = 1
GEMM_ERR_UNSUPPORTED = 2
GEMM_ERR_CUDA = 3
GEMM_ERR_TIMEOUT = 4
GEMM_ERR_NO_MEMORY = 5

GEMM_OUT_F32 = 0
GEMM_OUT_BF16 = 1

# Every function declared in include/gemm_bf16.h: (restype, argtypes).
_I = ctypes.c_int
_LL = ctypes.c_longlong
_F = ctypes.c_float
_P = ctypes.c_void_p
SIGNATURES = {
    "gemm_bf16": (_I, [_I, _I, _I, _P, _I, _P, _I, _P, _I, _I, _F, _F, _P]),
    "gemm_bf16_batched_shared_w": (_I, [_I, _I, _I, _I, _P, _I, _P, _I, _LL, _P, _I, _LL, _I, _F, _F,
                                        _P]),
    "gemm_bf16_status_string": (ctypes.c_char_p, [_I]),
    "gemm_bf16_device_status": (_I, [_P]),
    "gemm_bf16_set_plan": (_I, [_I]),
    "gemm_bf16_set_wait_timeout_ns": (_I, [ctypes.c_ulonglong]),
    "gemm_bf16_version": (_I, []),
    "gemm_bf16_noalloc": (_I, [_I, _I, _I, _P, _I, _P, _I, _P, _I, _I, _F, _F, _P]),
}

# Size of the fixed device scratch used by gemm_bf16_noalloc (GEMM_BF16_NOALLOC_SCRATCH_BYTES).
GEMM_BF16_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class GemmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {status_string(status)}" if what else status_string(status))


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python dsl_persistent_warp_b200/_build.py` "
            "(there is no CPU or fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def gemm_bf16(M, N, K, A, lda, B, ldb, C, ldc, out_type, alpha, beta, stream) -> int:
    return LIB.gemm_bf16(M, N, K, A, lda, B, ldb, C, ldc, out_type, alpha, beta, stream)


def gemm_bf16_batched_shared_w(batch, M, N, K, W, ldw, X, ldx, stride_x, Y, ldy, stride_y, out_type,
                               alpha, beta, stream) -> int:
    return LIB.gemm_bf16_batched_shared_w(batch, M, N, K, W, ldw, X, ldx, stride_x, Y, ldy, stride_y,
                                          out_type, alpha, beta, stream)


def gemm_bf16_status_string(status) -> str:
    return LIB.gemm_bf16_status_string(int(status)).decode()


status_string = gemm_bf16_status_string


def gemm_bf16_device_status(stream) -> int:
    return LIB.gemm_bf16_device_status(stream)


def gemm_bf16_set_plan(plan: int) -> int:
    return LIB.gemm_bf16_set_plan(int(plan))


def gemm_bf16_set_wait_timeout_ns(ns: int) -> int:
    return LIB.gemm_bf16_set_wait_timeout_ns(int(ns))


def gemm_bf16_version() -> int:
    return LIB.gemm_bf16_version()


def gemm_bf16_noalloc(M, N, K, A, lda, B, ldb, C, ldc, out_type, alpha, beta, stream) -> int:
    """gemm_bf16 without any device allocation (fixed 32 MiB library scratch)."""
    return LIB.gemm_bf16_noalloc(M, N, K, A, lda, B, ldb, C, ldc, out_type, alpha, beta, stream)
