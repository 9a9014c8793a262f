"""Failure detection on the GPU without a fault: every barrier wait in the kernels is bounded.

With the test hook GEMM_BF16_TEST_STALL_LOADS=1 the producer issues no loads, so a barrier that
nothing completes makes the MMA thread's bounded wait expire.  The kernel must then record the
timeout, release its tensor memory and return; gemm_bf16_device_status reports
GEMM_ERR_TIMEOUT, and the same process goes on computing correct results.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from parity import check, to_dev_bf16, values_f64
from synth import matrix_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture
def capi():
    from dsl_persistent_warp_b200 import capi as c
    yield c
    for k in ("GEMM_BF16_TEST_STALL_LOADS", "GEMM_BF16_CLUSTER_SPLIT", "GEMM_BF16_SPLIT_K"):
        os.environ.pop(k, None)
    c.gemm_bf16_set_wait_timeout_ns(0)
    c.gemm_bf16_set_plan(-1)


# (plan, forced split): the persistent plans, and K cut across a cluster (every CTA of the cluster
# must still reach both cluster barriers) or through the workspace.
CASES = [(0, None), (2, None), (4, None), (5, None), (1, ("GEMM_BF16_CLUSTER_SPLIT", "2")),
         (0, ("GEMM_BF16_CLUSTER_SPLIT", "4")), (2, ("GEMM_BF16_CLUSTER_SPLIT", "2")),
         (3, ("GEMM_BF16_CLUSTER_SPLIT", "4")), (0, ("GEMM_BF16_SPLIT_K", "2"))]


@pytest.mark.parametrize("case", CASES, ids=[f"plan{p}" + (f"_{e[0][10:]}{e[1]}" if e else "") for p, e in CASES])
def test_expired_wait_reports_timeout_and_context_survives(capi, case):
    plan, split = case
    if split:
        os.environ[split[0]] = split[1]
    import dsl_persistent_warp_b200 as pw
    M = N = K = 512
    A = matrix_bf16(71, M, K)
    B = matrix_bf16(72, N, K)
    dA, dB = to_dev_bf16(A), to_dev_bf16(B)
    s = torch.cuda.current_stream().cuda_stream
    assert capi.gemm_bf16_set_plan(plan) == 0
    assert capi.gemm_bf16_device_status(s) == capi.GEMM_OK  # nothing pending

    capi.gemm_bf16_set_wait_timeout_ns(50_000_000)  # 50 ms
    os.environ["GEMM_BF16_TEST_STALL_LOADS"] = "1"
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    pw.gemm_bf16(dA, dB, C)
    assert capi.gemm_bf16_device_status(s) == capi.GEMM_ERR_TIMEOUT
    assert capi.gemm_bf16_device_status(s) == capi.GEMM_OK  # the word was cleared

    os.environ.pop("GEMM_BF16_TEST_STALL_LOADS")
    capi.gemm_bf16_set_wait_timeout_ns(0)
    pw.gemm_bf16(dA, dB, C)
    assert capi.gemm_bf16_device_status(s) == capi.GEMM_OK
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K)
    assert check(values_f64(C), Cref, R, out_bf16=False)["ok"]
