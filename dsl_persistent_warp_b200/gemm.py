"""PyTorch-facing wrappers of the C ABI: torch supplies device memory, pointers, strides and the
current stream; every step of the computation runs in the library's kernels.

    C = alpha * A @ B_stored.T + beta * C          gemm_bf16(A, B_stored, C)
    Y[b] = alpha * W @ X[b] + beta * Y[b]          gemm_bf16_batched_shared_w(W, X, Y)

A and B (W and X) may be bfloat16 or float16 (both the same type); the matching C entry point
(gemm_bf16* or gemm_f16*) is called.  C may be float32, bfloat16 or float16.
"""
from __future__ import annotations

import torch

from . import capi

_OUT = {torch.float32: capi.GEMM_OUT_F32, torch.bfloat16: capi.GEMM_OUT_BF16,
        torch.float16: capi.GEMM_OUT_F16}
_IN = (torch.bfloat16, torch.float16)


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _check(status: int, what: str):
    if status != capi.GEMM_OK:
        raise capi.GemmError(status, what)


def _rowmajor_2d(t: torch.Tensor, name: str):
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be a 2-D row-major tensor (unit column stride)")
    return max(int(t.stride(0)), 1) if t.shape[0] > 1 else max(int(t.shape[1]), 1)


def gemm_bf16(A: torch.Tensor, B: torch.Tensor, C: torch.Tensor | None = None, *, alpha: float = 1.0,
              beta: float = 0.0, out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """C = alpha * A @ B.T + beta * C for A (M x K) and B stored N x K ("K-major"), both bf16
    (or both fp16) CUDA tensors with unit column stride.  C (M x N, float32, bfloat16 or
    float16) is updated in place and returned; when omitted it is allocated (beta must then
    be 0)."""
    if A.dtype not in _IN or B.dtype != A.dtype:
        raise TypeError("A and B must both be bfloat16 or both float16")
    M, K = A.shape
    N, K2 = B.shape
    if K2 != K:
        raise ValueError("A and B disagree on K")
    if C is None:
        if beta != 0.0:
            raise ValueError("beta != 0 needs C")
        C = torch.empty((M, N), dtype=out_dtype, device=A.device)
    if C.shape != (M, N) or C.dtype not in _OUT:
        raise ValueError("C must be M x N float32/bfloat16/float16")
    lda = _rowmajor_2d(A, "A") if K else 1
    ldb = _rowmajor_2d(B, "B") if K else 1
    ldc = _rowmajor_2d(C, "C")
    fn = capi.gemm_f16 if A.dtype == torch.float16 else capi.gemm_bf16
    st = fn(M, N, K, A.data_ptr(), max(lda, K, 1), B.data_ptr(), max(ldb, K, 1),
                        C.data_ptr(), max(ldc, N, 1), _OUT[C.dtype], float(alpha), float(beta),
                        _stream_handle(stream))
    _check(st, fn.__name__)
    return C


def gemm_bf16_batched_shared_w(W: torch.Tensor, X: torch.Tensor, Y: torch.Tensor | None = None, *,
                               alpha: float = 1.0, beta: float = 0.0,
                               out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """Y[b] = alpha * W @ X[b] + beta * Y[b] for W (M x K, shared), X (batch x K x N) and
    Y (batch x M x N), all with unit innermost stride."""
    if W.dtype not in _IN or X.dtype != W.dtype:
        raise TypeError("W and X must both be bfloat16 or both float16")
    M, K = W.shape
    batch, K2, N = X.shape
    if K2 != K:
        raise ValueError("W and X disagree on K")
    if Y is None:
        if beta != 0.0:
            raise ValueError("beta != 0 needs Y")
        Y = torch.empty((batch, M, N), dtype=out_dtype, device=W.device)
    if Y.shape != (batch, M, N) or Y.dtype not in _OUT:
        raise ValueError("Y must be batch x M x N float32/bfloat16/float16")
    if (N > 1 and X.stride(2) != 1) or (N > 1 and Y.stride(2) != 1):
        raise ValueError("X and Y need unit innermost stride")
    ldw = _rowmajor_2d(W, "W") if K else 1
    fn = capi.gemm_f16_batched_shared_w if W.dtype == torch.float16 else capi.gemm_bf16_batched_shared_w
    st = fn(
        batch, M, N, K, W.data_ptr(), max(ldw, K, 1), X.data_ptr(), max(int(X.stride(1)), N, 1),
        int(X.stride(0)), Y.data_ptr(), max(int(Y.stride(1)), N, 1), int(Y.stride(0)), _OUT[Y.dtype],
        float(alpha), float(beta), _stream_handle(stream))
    _check(st, fn.__name__)
    return Y


def gemm_bf16_batched_shared_w_dedup(W: torch.Tensor, X: torch.Tensor, index: torch.Tensor,
                                     Y: torch.Tensor | None = None, *, alpha: float = 1.0, beta: float = 0.0,
                                     out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """Y[b] = alpha * W @ X[index[b]] + beta * Y[b] for W (M x K, shared), X (n_unique x K x N:
    the distinct entries) and index (batch int32 CUDA tensor); Y is batch x M x N."""
    if W.dtype != torch.bfloat16 or X.dtype != torch.bfloat16:
        raise TypeError("W and X must be bfloat16")
    if index.dtype != torch.int32 or index.dim() != 1 or not index.is_contiguous():
        raise TypeError("index must be a contiguous 1-D int32 tensor")
    M, K = W.shape
    n_unique, K2, N = X.shape
    if K2 != K:
        raise ValueError("W and X disagree on K")
    batch = int(index.shape[0])
    if Y is None:
        if beta != 0.0:
            raise ValueError("beta != 0 needs Y")
        Y = torch.empty((batch, M, N), dtype=out_dtype, device=W.device)
    if Y.shape != (batch, M, N) or Y.dtype not in _OUT:
        raise ValueError("Y must be batch x M x N float32/bfloat16/float16")
    if (N > 1 and X.stride(2) != 1) or (N > 1 and Y.stride(2) != 1):
        raise ValueError("X and Y need unit innermost stride")
    ldw = _rowmajor_2d(W, "W") if K else 1
    st = capi.gemm_bf16_batched_shared_w_dedup(
        batch, n_unique, M, N, K, W.data_ptr(), max(ldw, K, 1), X.data_ptr(), max(int(X.stride(1)), N, 1),
        int(X.stride(0)), index.data_ptr(), Y.data_ptr(), max(int(Y.stride(1)), N, 1), int(Y.stride(0)),
        _OUT[Y.dtype], float(alpha), float(beta), _stream_handle(stream))
    _check(st, "gemm_bf16_batched_shared_w_dedup")
    return Y


def device_status(stream=None) -> int:
    """Synchronize the stream and return the library's device status (GEMM_OK / TIMEOUT)."""
    return capi.gemm_bf16_device_status(_stream_handle(stream))
