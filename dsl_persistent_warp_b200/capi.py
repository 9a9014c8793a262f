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
GEMM_OUT_F16 = 2

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
    "gemm_f16": (_I, [_I, _I, _I, _P, _I, _P, _I, _P, _I, _I, _F, _F, _P]),
    "gemm_f16_batched_shared_w": (_I, [_I, _I, _I, _I, _P, _I, _P, _I, _LL, _P, _I, _LL, _I, _F, _F,
                                       _P]),
    "gemm_bf16_batched_shared_w_dedup": (_I, [_I, _I, _I, _I, _I, _P, _I, _P, _I, _LL, _P, _P, _I, _LL, _I,
                                              _F, _F, _P]),
    "gemm_autotune": (_I, [_I, _I, _I, _I, _I, _I, _I, _P, _I, _P, _I, _LL, _P, _P, _I, _LL, _I, _F, _F, _P,
                           ctypes.POINTER(ctypes.c_float)]),
    "gemm_tuning_clear": (_I, []),
    "gemm_tuning_size": (_I, []),
    "gemm_tuning_save": (_I, [ctypes.c_char_p]),
    "gemm_tuning_load": (_I, [ctypes.c_char_p]),
    "gemm_last_config": (_I, [ctypes.POINTER(_I)] * 4),
    "gemm_bf16_tensor_map_cache_stats": (_I, [ctypes.POINTER(ctypes.c_ulonglong),
                                              ctypes.POINTER(ctypes.c_ulonglong)]),
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


def gemm_f16(M, N, K, A, lda, B, ldb, C, ldc, out_type, alpha, beta, stream) -> int:
    return LIB.gemm_f16(M, N, K, A, lda, B, ldb, C, ldc, out_type, alpha, beta, stream)


def gemm_f16_batched_shared_w(batch, M, N, K, W, ldw, X, ldx, stride_x, Y, ldy, stride_y, out_type,
                              alpha, beta, stream) -> int:
    return LIB.gemm_f16_batched_shared_w(batch, M, N, K, W, ldw, X, ldx, stride_x, Y, ldy, stride_y,
                                         out_type, alpha, beta, stream)


def gemm_bf16_tensor_map_cache_stats() -> tuple[int, int]:
    """(hits, misses) of the library's tensor-map cache."""
    h, m = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    st = LIB.gemm_bf16_tensor_map_cache_stats(ctypes.byref(h), ctypes.byref(m))
    if st != GEMM_OK:
        raise GemmError(st, "gemm_bf16_tensor_map_cache_stats")
    return int(h.value), int(m.value)


def gemm_bf16_batched_shared_w_dedup(batch, n_unique, M, N, K, W, ldw, X, ldx, stride_x, index, Y, ldy,
                                     stride_y, out_type, alpha, beta, stream) -> int:
    return LIB.gemm_bf16_batched_shared_w_dedup(batch, n_unique, M, N, K, W, ldw, X, ldx, stride_x, index,
                                                Y, ldy, stride_y, out_type, alpha, beta, stream)


def gemm_autotune(in_type, form, batch, n_unique, M, N, K, A, lda, B, ldb, stride_b, index, C, ldc, stride_c,
                  out_type, alpha, beta, stream) -> tuple[int, float]:
    """(status, best time per call in us) of the C autotuner."""
    best = ctypes.c_float(0.0)
    st = LIB.gemm_autotune(in_type, form, batch, n_unique, M, N, K, A, lda, B, ldb, stride_b, index, C, ldc,
                           stride_c, out_type, alpha, beta, stream, ctypes.byref(best))
    return st, float(best.value)


def gemm_tuning_clear() -> int:
    return LIB.gemm_tuning_clear()


def gemm_tuning_size() -> int:
    return LIB.gemm_tuning_size()


def gemm_tuning_save(path: str) -> int:
    return LIB.gemm_tuning_save(path.encode())


def gemm_tuning_load(path: str) -> int:
    return LIB.gemm_tuning_load(path.encode())


def gemm_last_config() -> tuple[int, int, int, int]:
    """(plan, workspace K slices (0: stream-K), cluster K slices, raster group) of this thread's
    last launch."""
    v = [ctypes.c_int(0) for _ in range(4)]
    st = LIB.gemm_last_config(*[ctypes.byref(x) for x in v])
    if st != GEMM_OK:
        raise GemmError(st, "gemm_last_config")
    return tuple(int(x.value) for x in v)
