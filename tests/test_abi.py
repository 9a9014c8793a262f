"""The C-ABI library on the CPU: it loads, exports every symbol include/gemm_bf16.h declares,
and rejects bad arguments before touching CUDA.  No compute call runs here."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gemm_bf16.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"GEMM_API\s+[\w\s\*]+?\b(gemm_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def capi():
    from conftest import build_library
    build_library()
    from dsl_persistent_warp_b200 import capi as c
    return c


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("gemm_bf16", "gemm_bf16_batched_shared_w", "gemm_bf16_status_string",
                     "gemm_f16", "gemm_f16_batched_shared_w"):
        assert required in names


def test_library_exports_every_declared_symbol(capi):
    out = subprocess.run(["nm", "-D", "--defined-only", capi.LIB._name], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)$", out, flags=re.M))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    # the binding covers exactly the declared functions, under the same names
    assert sorted(capi.SIGNATURES) == _declared_functions()
    # nothing beyond the boundary leaks out of the library
    extra = sorted(n for n in exported if n.startswith("gemm") and n not in capi.SIGNATURES)
    assert not extra, extra


def test_status_strings(capi):
    assert capi.gemm_bf16_status_string(0) == "GEMM_OK"
    assert capi.gemm_bf16_status_string(4) == "GEMM_ERR_TIMEOUT"
    assert capi.gemm_bf16_status_string(99) == "GEMM_ERR_UNKNOWN"
    assert capi.gemm_bf16_version() >= 100


BAD_GEMM_CALLS = [
    # (M, N, K, A, lda, B, ldb, C, ldc, out, alpha, beta)
    (-1, 4, 4, 16, 4, 16, 4, 16, 4, 1, 1.0, 0.0),   # negative M
    (4, -2, 4, 16, 4, 16, 4, 16, 4, 1, 1.0, 0.0),   # negative N
    (4, 4, -3, 16, 4, 16, 4, 16, 4, 1, 1.0, 0.0),   # negative K
    (4, 4, 8, 16, 7, 16, 8, 16, 4, 1, 1.0, 0.0),    # lda < K
    (4, 4, 8, 16, 8, 16, 7, 16, 4, 1, 1.0, 0.0),    # ldb < K
    (4, 4, 8, 16, 8, 16, 8, 16, 3, 1, 1.0, 0.0),    # ldc < N
    (4, 4, 8, 16, 8, 16, 8, 16, 4, 3, 1.0, 0.0),    # unknown out_type
    (4, 4, 8, 16, 8, 16, 8, 17, 4, 2, 1.0, 0.0),    # fp16 C not 2-byte aligned
    (4, 4, 8, 16, 8, 16, 8, None, 4, 1, 1.0, 0.0),  # NULL C
    (4, 4, 8, None, 8, 16, 8, 16, 4, 1, 1.0, 0.0),  # NULL A with work to do
    (4, 4, 8, 16, 8, None, 8, 16, 4, 1, 1.0, 0.0),  # NULL B with work to do
    (4, 4, 8, 17, 8, 16, 8, 16, 4, 1, 1.0, 0.0),    # A not 2-byte aligned
    (4, 4, 8, 16, 8, 16, 8, 18, 4, 0, 1.0, 0.0),    # fp32 C not 4-byte aligned
]


@pytest.mark.parametrize("args", BAD_GEMM_CALLS)
@pytest.mark.parametrize("entry", ["gemm_bf16", "gemm_f16", "gemm_bf16_noalloc"])
def test_gemm_rejects_bad_arguments(capi, args, entry):
    assert getattr(capi, entry)(*args, None) == capi.GEMM_ERR_INVALID_ARG


def test_empty_problems_are_ok_without_a_device(capi):
    assert capi.gemm_bf16(0, 4, 4, None, 4, None, 4, None, 4, 1, 1.0, 0.0, None) == capi.GEMM_OK
    assert capi.gemm_bf16(4, 0, 4, None, 4, None, 4, None, 1, 1, 1.0, 0.0, None) == capi.GEMM_OK
    assert capi.gemm_bf16_batched_shared_w(0, 4, 4, 4, None, 4, None, 4, 16, None, 4, 16, 1, 1.0,
                                           0.0, None) == capi.GEMM_OK


BAD_BATCHED = [
    # (batch, M, N, K, W, ldw, X, ldx, stride_x, Y, ldy, stride_y, out, alpha, beta)
    (-1, 4, 4, 4, 16, 4, 16, 4, 16, 16, 4, 16, 1, 1.0, 0.0),   # negative batch
    (2, 4, 4, 4, 16, 4, 16, 3, 16, 16, 4, 16, 1, 1.0, 0.0),    # ldx < N
    (2, 4, 4, 4, 16, 4, 16, 4, -1, 16, 4, 16, 1, 1.0, 0.0),    # negative stride_x
    (2, 4, 4, 4, 16, 4, 16, 4, 16, 16, 4, 8, 1, 1.0, 0.0),     # output batches overlap
    (2, 4, 4, 4, 16, 3, 16, 4, 16, 16, 4, 16, 1, 1.0, 0.0),    # ldw < K
]


@pytest.mark.parametrize("args", BAD_BATCHED)
@pytest.mark.parametrize("entry", ["gemm_bf16_batched_shared_w", "gemm_f16_batched_shared_w"])
def test_batched_rejects_bad_arguments(capi, args, entry):
    assert getattr(capi, entry)(*args, None) == capi.GEMM_ERR_INVALID_ARG


def test_tensor_map_cache_stats_without_a_device(capi):
    """No call has reached the encoder in a process without a GPU: the cache is empty."""
    assert capi.gemm_bf16_tensor_map_cache_stats() == (0, 0)
    assert capi.LIB.gemm_bf16_tensor_map_cache_stats(None, None) == capi.GEMM_ERR_INVALID_ARG


def test_set_plan_and_timeout(capi):
    assert capi.gemm_bf16_set_plan(9) == capi.GEMM_ERR_INVALID_ARG
    assert capi.gemm_bf16_set_plan(-2) == capi.GEMM_ERR_INVALID_ARG
    for p in (0, 1, 2, 3, 4, 5, 6, 7, 8, -1):
        assert capi.gemm_bf16_set_plan(p) == capi.GEMM_OK
    assert capi.gemm_bf16_set_wait_timeout_ns(0) == capi.GEMM_OK


def test_library_links_no_torch():
    """The boundary is plain C: the shared library depends on no PyTorch library."""
    from conftest import build_library
    path = build_library()
    out = subprocess.run(["ldd", path], capture_output=True, text=True).stdout
    assert "torch" not in out and "c10" not in out
