"""gemm_bf16_noalloc: the allocation-free entry point, for callers that cannot let a library
allocate device memory (their memory is handed out by their own allocator or budget, or the
call sits on a latency-critical path).  It must give the same results as gemm_bf16 while
keeping its pre-pass copies in the library's fixed device scratch.

This file is collected last on purpose; it passes alone in a fresh process and after the other
tests.  Every call goes through the C ABI (ctypes)."""
import numpy as np
import pytest
import torch

import oracle
from parity import check, to_dev_bf16, values_f64
from synth import matrix_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def capi():
    from dsl_persistent_warp_b200 import capi as c
    c.gemm_bf16_set_plan(-1)
    return c


def _call(fn, capi, dA, lda, dB, ldb, M, N, K, out, alpha, beta, c0):
    C = c0.clone()
    st = fn(M, N, K, dA.data_ptr(), lda, dB.data_ptr(), ldb, C.data_ptr(), N,
            capi.GEMM_OUT_BF16 if out == torch.bfloat16 else capi.GEMM_OUT_F32, alpha, beta,
            torch.cuda.current_stream().cuda_stream)
    assert st == capi.GEMM_OK, capi.gemm_bf16_status_string(st)
    return C


# Two calls in a row with different operands; both need the alignment pre-pass (packed,
# odd leading dimensions), so both go through the scratch.
CASES = [
    # M, N, K, out, alpha, beta
    (301, 263, 1003, torch.bfloat16, 0.5, 1.0),
    (517, 136, 771, torch.float32, 1.0, 0.0),
]


def test_noalloc_matches_gemm_bf16_on_consecutive_calls(capi):
    for i, (M, N, K, out, alpha, beta) in enumerate(CASES):
        A = matrix_bf16(900 + 3 * i, M, K)  # lda = K: not a multiple of 8
        B = matrix_bf16(901 + 3 * i, N, K)
        dA, dB = to_dev_bf16(A), to_dev_bf16(B)
        c0 = torch.randn(M, N, device="cuda").to(out)
        ref = _call(capi.gemm_bf16, capi, dA, K, dB, K, M, N, K, out, alpha, beta, c0)
        got = _call(capi.gemm_bf16_noalloc, capi, dA, K, dB, K, M, N, K, out, alpha, beta, c0)
        torch.cuda.synchronize()
        assert capi.gemm_bf16_device_status(torch.cuda.current_stream().cuda_stream) == 0
        # tolerance of the parity tests, with the bound R of these inputs from the oracle
        _, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0.float().cpu().numpy(), alpha=alpha,
                           beta=beta)
        rep = check(values_f64(got), values_f64(ref), R, out_bf16=out == torch.bfloat16)
        assert rep["ok"], (i, rep)


def test_noalloc_rejects_problems_beyond_its_scratch(capi):
    # 4099 x 4099 packed A and B need ~67 MB of padded copies: more than the 32 MiB scratch.
    n = 4099
    assert 2 * n * (n + 5) * 2 > capi.GEMM_BF16_NOALLOC_SCRATCH_BYTES
    dA = torch.zeros(n * n, dtype=torch.bfloat16, device="cuda")
    C = torch.full((n, n), 7.0, dtype=torch.bfloat16, device="cuda")
    st = capi.gemm_bf16_noalloc(n, n, n, dA.data_ptr(), n, dA.data_ptr(), n, C.data_ptr(), n,
                                capi.GEMM_OUT_BF16, 1.0, 0.0,
                                torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == capi.GEMM_ERR_INVALID_ARG
    assert bool((C == 7.0).all())  # nothing was enqueued
