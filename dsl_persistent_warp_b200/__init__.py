"""B200-native (sm_100a) persistent, warp-specialized BF16 GEMM behind a C ABI.

``capi`` holds the ctypes binding of include/gemm_bf16.h under the C names; ``gemm`` holds
thin PyTorch wrappers (torch supplies memory, pointers and streams only).
"""
from . import capi  # noqa: F401  (raises ImportError when the CUDA library is missing)
from .gemm import (device_status, gemm_bf16, gemm_bf16_batched_shared_w,  # noqa: F401
                   gemm_bf16_batched_shared_w_dedup)

__all__ = ["capi", "gemm_bf16", "gemm_bf16_batched_shared_w", "gemm_bf16_batched_shared_w_dedup",
           "device_status"]
