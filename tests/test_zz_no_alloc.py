"""gemm_bf16_noalloc: the allocation-free entry point, for callers that cannot let a library
allocate device memory (their memory is handed out by their own allocator or budget, or the
call sits on a latency-critical path).  Its results must match the fp64 oracle within the
parity tests' tolerance while its pre-pass copies live in the library's fixed device scratch,
and a warmed-up call must not change the device's free memory.

The file name sorts last so that a run stopping at its first failure has already run every
other test; nothing here depends on the order (it passes alone in a fresh process and after the
other tests).  Every call goes through the C ABI (ctypes)."""
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


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _call(fn, capi, dA, lda, dB, ldb, M, N, K, out, alpha, beta, C):
    st = fn(M, N, K, dA.data_ptr(), lda, dB.data_ptr(), ldb, C.data_ptr(), N,
            capi.GEMM_OUT_BF16 if out == torch.bfloat16 else capi.GEMM_OUT_F32, alpha, beta, _stream())
    assert st == capi.GEMM_OK, capi.gemm_bf16_status_string(st)


# Two calls in a row with different operands; both need the alignment pre-pass (packed,
# odd leading dimensions), so both go through the scratch and the second overwrites the first's
# copies.
CASES = [
    # M, N, K, out, alpha, beta
    (301, 263, 1003, torch.bfloat16, 0.5, 1.0),
    (517, 136, 771, torch.float32, 1.0, 0.0),
]


def test_noalloc_matches_the_oracle_on_consecutive_calls(capi):
    for i, (M, N, K, out, alpha, beta) in enumerate(CASES):
        A = matrix_bf16(900 + 3 * i, M, K)  # lda = K: not a multiple of 8
        B = matrix_bf16(901 + 3 * i, N, K)
        c0bits = matrix_bf16(902 + 3 * i, M, N)
        dA, dB = to_dev_bf16(A), to_dev_bf16(B)
        C = to_dev_bf16(c0bits).to(out)
        _call(capi.gemm_bf16_noalloc, capi, dA, K, dB, K, M, N, K, out, alpha, beta, C)
        torch.cuda.synchronize()
        assert capi.gemm_bf16_device_status(_stream()) == 0
        Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits if beta != 0.0 else None, alpha=alpha,
                              beta=beta)
        rep = check(values_f64(C), Cref, R, out_bf16=out == torch.bfloat16)
        assert rep["ok"], (i, rep)


def test_noalloc_takes_no_device_memory(capi):
    """After one warm-up call (which may load the library's kernels and look up the scratch's
    address), further calls leave the device's free memory exactly as it was."""
    M, N, K = 301, 263, 1003
    dA, dB = to_dev_bf16(matrix_bf16(910, M, K)), to_dev_bf16(matrix_bf16(911, N, K))
    C = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    _call(capi.gemm_bf16_noalloc, capi, dA, K, dB, K, M, N, K, torch.bfloat16, 1.0, 0.0, C)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        _call(capi.gemm_bf16_noalloc, capi, dA, K, dB, K, M, N, K, torch.bfloat16, 1.0, 0.0, C)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_cuts_deep_k_across_a_cluster(capi):
    """A few-tile, deep-K problem: the allocation-free entry point may still cut K, across the
    CTAs of a cluster (partial sums exchanged in shared memory, no memory needed)."""
    M, N, K = 512, 512, 8192
    A, B = matrix_bf16(920, M, K, std=K ** -0.5), matrix_bf16(921, N, K)
    dA, dB = to_dev_bf16(A), to_dev_bf16(B)
    C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    _call(capi.gemm_bf16_noalloc, capi, dA, K, dB, K, M, N, K, torch.float32, 1.0, 0.0, C)
    torch.cuda.synchronize()
    assert capi.gemm_bf16_device_status(_stream()) == 0
    plan, splits, csplit, _ = capi.gemm_last_config()
    assert splits == 1 and csplit > 1, (plan, splits, csplit)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K)
    assert check(values_f64(C), Cref, R, out_bf16=False)["ok"]


def test_noalloc_rejects_problems_beyond_its_scratch(capi):
    # 4099 x 4099 packed A and B need ~67 MB of padded copies: more than the 32 MiB scratch.
    n = 4099
    assert 2 * n * (n + 5) * 2 > capi.GEMM_BF16_NOALLOC_SCRATCH_BYTES
    dA = torch.zeros(n * n, dtype=torch.bfloat16, device="cuda")
    C = torch.full((n, n), 7.0, dtype=torch.bfloat16, device="cuda")
    st = capi.gemm_bf16_noalloc(n, n, n, dA.data_ptr(), n, dA.data_ptr(), n, C.data_ptr(), n,
                                capi.GEMM_OUT_BF16, 1.0, 0.0, _stream())
    torch.cuda.synchronize()
    assert st == capi.GEMM_ERR_INVALID_ARG
    assert bool((C == 7.0).all())  # nothing was enqueued
