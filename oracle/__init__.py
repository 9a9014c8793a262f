"""TEST INFRASTRUCTURE ONLY: the fp64 CPU oracle of C = alpha*A*B + beta*C.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The GPU product path never does: it shares no code with this module
and fails loudly when its CUDA library is missing.

The arithmetic lives in ``gemm_ref.c`` (plain C, float64, k ascending); this file only
compiles it with gcc and marshals numpy arrays through ctypes.  Every result is
``(Cref, R)``: the float64 reference values and the magnitude bound
R = |alpha| * sum_k |a||b| + |beta| * |c0| used by the tolerances.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gemm_ref.c")
_LIB_NAME = "liboracle_gemm.so"
_lock = threading.Lock()
_libs: dict[int, ctypes.CDLL] = {}


def build(plant: int = 0, out_dir: str | None = None) -> str:
    """Compile gemm_ref.c (gcc -O2 -fopenmp, no fast-math).  ``plant`` != 0 builds a copy
    with one deliberate mistake (for the tests that show the pins catch it)."""
    out_dir = out_dir or _HERE
    name = _LIB_NAME if plant == 0 else f"liboracle_gemm_plant{plant}.so"
    out = os.path.join(out_dir, name)
    if (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-shared",
               "-fPIC", f"-DORACLE_PLANT={int(plant)}", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _lib(plant: int = 0, out_dir: str | None = None) -> ctypes.CDLL:
    key = plant if out_dir is None else hash((plant, out_dir))
    with _lock:
        if key not in _libs:
            lib = ctypes.CDLL(build(plant, out_dir))
            P = ctypes.c_void_p
            LL = ctypes.c_longlong
            I = ctypes.c_int
            D = ctypes.c_double
            lib.oracle_gemm.argtypes = [I, I, I, P, LL, P, LL, I, P, LL, I, D, D, P, I, P, P, I]
            lib.oracle_gemm.restype = I
            lib.oracle_gemm_batched.argtypes = [I, I, I, I, P, LL, P, LL, LL, P, LL, LL, I, D,
                                                D, P, I, P, P, I, P, I]
            lib.oracle_decode.argtypes = [I, P, LL, P]
            lib.oracle_decode.restype = None
            lib.oracle_gemm_batched.restype = I
            lib.oracle_threads.restype = I
            lib.oracle_plant.restype = I
            _libs[key] = lib
        return _libs[key]


def threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else the host's cores)."""
    return int(_lib().oracle_threads())


def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c0_type(c0: np.ndarray | None) -> int:
    if c0 is None:
        return 0
    if c0.dtype == np.float32:
        return 1
    if c0.dtype == np.uint16:
        return 2
    if c0.dtype == np.float16:
        return 3
    raise TypeError("c0 must be float32, uint16 (bfloat16 bits) or float16")


_IN_TYPES = {"bf16": 0, "f16": 1}


def _in_type(A: np.ndarray, in_dtype: str | None) -> int:
    """16-bit operand type: explicit ``in_dtype`` ('bf16' / 'f16'), else fp16 for float16
    arrays and bf16 for uint16 bit patterns."""
    if in_dtype is not None:
        return _IN_TYPES[in_dtype]
    return 1 if A.dtype == np.float16 else 0


def _bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    return np.ascontiguousarray(a, dtype=np.uint16)


def decode(h: np.ndarray, in_dtype: str, plant: int = 0, lib_dir: str | None = None) -> np.ndarray:
    """Exact float64 values of 16-bit patterns ('bf16' or 'f16'), decoded by the oracle."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float64)
    _lib(plant, lib_dir).oracle_decode(_IN_TYPES[in_dtype], _ptr(h), int(h.size), _ptr(out))
    return out


def gemm(A: np.ndarray, B: np.ndarray, *, M: int, N: int, K: int, b_kmajor: bool = True,
         c0: np.ndarray | None = None, alpha: float = 1.0, beta: float = 0.0,
         rows=None, plant: int = 0, lib_dir: str | None = None, in_dtype: str | None = None):
    """Reference rows of C = alpha*A*B + beta*c0.

    A: 2-D, M x lda with lda >= K: uint16 bit patterns (bf16 unless ``in_dtype`` = 'f16') or
       float16.  B: the same type, 2-D; N x ldb (K-major, ``b_kmajor``) or K x ldb (N-major).
    c0: None, or float32 / uint16 (bf16 bits) / float16 2-D M x ldc.
    rows: None (all M rows) or a sequence of row indices.
    Returns (Cref, R), float64 arrays of shape (len(rows), N).
    """
    it = _in_type(A, in_dtype)
    A = _bits(A)
    B = _bits(B)
    lda = A.shape[1] if A.ndim == 2 and A.size else max(K, 1)
    ldb = B.shape[1] if B.ndim == 2 and B.size else max(K if b_kmajor else N, 1)
    if M and K:
        assert A.shape[0] >= M and lda >= K
    if N and K:
        assert B.shape[0] >= (N if b_kmajor else K) and ldb >= (K if b_kmajor else N)
    ldc = 0
    if c0 is not None:
        c0 = np.ascontiguousarray(c0)
        ldc = c0.shape[1]
        assert c0.shape[0] >= M and ldc >= N
    if rows is None:
        rows_arr = None
        nrows = M
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        assert rows_arr.size == 0 or (rows_arr.min() >= 0 and rows_arr.max() < M)
        nrows = int(rows_arr.size)
    Cref = np.empty((nrows, N), dtype=np.float64)
    R = np.empty((nrows, N), dtype=np.float64)
    rc = _lib(plant, lib_dir).oracle_gemm(
        M, N, K, _ptr(A), lda, _ptr(B), ldb, 1 if b_kmajor else 0, _ptr(c0), ldc,
        _c0_type(c0), float(alpha), float(beta), _ptr(rows_arr), nrows, _ptr(Cref), _ptr(R), it)
    if rc != 0:
        raise ValueError("oracle_gemm rejected its arguments")
    return Cref, R


def gemm_batched(W: np.ndarray, X: np.ndarray, *, batch: int, M: int, N: int, K: int,
                 stride_x: int, y0: np.ndarray | None = None, stride_y: int = 0,
                 alpha: float = 1.0, beta: float = 0.0, rows=None, plant: int = 0,
                 lib_dir: str | None = None, in_dtype: str | None = None):
    """Reference of Y[b] = alpha*W*X[b] + beta*Y0[b] for every b < batch.

    W: 2-D M x ldw, uint16 bit patterns (bf16 unless ``in_dtype`` = 'f16') or float16.
    X: the same type, 1-D or 2-D buffer; X[b] starts at element b*stride_x
    and is K x N row-major with ldx = X.shape[-1] when 2-D (pass 2-D as (batch*K, ldx) or
    (batch*K_pad, ldx)).  y0: None or float32/uint16/float16 buffer laid out like Y, 2-D
    (rows, ldy).
    Returns (Cref, R) of shape (batch, len(rows), N).
    """
    it = _in_type(W, in_dtype)
    W = _bits(W)
    X = _bits(X)
    ldw = W.shape[1]
    ldx = X.shape[-1]
    ldy = 0
    if y0 is not None:
        y0 = np.ascontiguousarray(y0)
        ldy = y0.shape[-1]
    if rows is None:
        rows_arr = None
        nrows = M
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        nrows = int(rows_arr.size)
    Cref = np.empty((batch, nrows, N), dtype=np.float64)
    R = np.empty((batch, nrows, N), dtype=np.float64)
    rc = _lib(plant, lib_dir).oracle_gemm_batched(
        batch, M, N, K, _ptr(W), ldw, _ptr(X), ldx, int(stride_x), _ptr(y0), ldy,
        int(stride_y), _c0_type(y0), float(alpha), float(beta), _ptr(rows_arr), nrows,
        _ptr(Cref), _ptr(R), it, None, 0)
    if rc != 0:
        raise ValueError("oracle_gemm_batched rejected its arguments")
    return Cref, R


def gemm_batched_dedup(W: np.ndarray, X: np.ndarray, index, *, n_x: int, M: int, N: int, K: int,
                       stride_x: int, y0: np.ndarray | None = None, stride_y: int = 0,
                       alpha: float = 1.0, beta: float = 0.0, rows=None, plant: int = 0,
                       lib_dir: str | None = None, in_dtype: str | None = None):
    """Reference of Y[b] = alpha*W*X[index[b]] + beta*Y0[b] for every b < len(index): the
    deduplicated shared-W form, where X holds only the n_x distinct entries (X[u] starts at
    element u*stride_x, K x N row-major with ldx = X.shape[-1]) and item b uses entry index[b].
    Returns (Cref, R) of shape (len(index), len(rows), N)."""
    it = _in_type(W, in_dtype)
    W = _bits(W)
    X = _bits(X)
    idx = np.ascontiguousarray(np.asarray(index, dtype=np.int32))
    batch = int(idx.size)
    ldw = W.shape[1]
    ldx = X.shape[-1]
    ldy = 0
    if y0 is not None:
        y0 = np.ascontiguousarray(y0)
        ldy = y0.shape[-1]
    if rows is None:
        rows_arr = None
        nrows = M
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        nrows = int(rows_arr.size)
    Cref = np.empty((batch, nrows, N), dtype=np.float64)
    R = np.empty((batch, nrows, N), dtype=np.float64)
    rc = _lib(plant, lib_dir).oracle_gemm_batched(
        batch, M, N, K, _ptr(W), ldw, _ptr(X), ldx, int(stride_x), _ptr(y0), ldy,
        int(stride_y), _c0_type(y0), float(alpha), float(beta), _ptr(rows_arr), nrows,
        _ptr(Cref), _ptr(R), it, _ptr(idx), int(n_x))
    if rc != 0:
        raise ValueError("oracle_gemm_batched rejected its arguments (index out of range?)")
    return Cref, R
