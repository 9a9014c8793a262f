"""Stream-K: the tiles of the last, partial wave of the persistent walk are computed as K ranges
spread evenly over every cluster and added up by the split-K fixup.  Parity against the fp64
oracle (sampled rows at these sizes: every 128-row block, both tile borders, every epilogue
warp's lane quarter), bit-exact small-integer sums, and the same bits on a second call.
Every call goes through the C ABI; the configuration actually launched is read back with
gemm_last_config (stream-K reports 0 workspace slices)."""
import os

import numpy as np
import pytest
import torch

import oracle
from parity import bits_of, check, sample_rows, to_dev_bf16, to_dev_f16, values_f64
from synth import bf16_bits_to_f64, f64_to_bf16_bits, matrix_bf16, matrix_f16

pytestmark = pytest.mark.gpu

# plan -> (M, N, K): more tiles than the plan has persistent clusters on a 148-SM B200, a
# partial last wave, and a K long enough for ranges of at least 8 k-blocks; ragged M, N and K.
CASES = {
    4: (4000, 4090, 1000),   # 256x512 tiles on CTA pairs, two MMA sub-tiles
    2: (2500, 2560, 1500),   # 256x256 on CTA pairs
    3: (2304, 1152, 5500),   # 256x128 on CTA pairs
    0: (1664, 1600, 7000),   # 128x128
    1: (2560, 2048, 6400),   # 128x256
    8: (1200, 1000, 6400),   # 128x64
}


@pytest.fixture()
def pw():
    import dsl_persistent_warp_b200 as m
    os.environ["GEMM_BF16_STREAM_K"] = "1"
    yield m
    os.environ.pop("GEMM_BF16_STREAM_K", None)
    m.capi.gemm_bf16_set_plan(-1)


def _launch(pw, A, B, M, N, K, out, alpha, beta, c0=None):
    C = torch.empty((M, N), dtype=out, device="cuda") if c0 is None else c0.to(out).cuda()
    pw.gemm_bf16(to_dev_bf16(A), to_dev_bf16(B), C, alpha=alpha, beta=beta)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    plan, splits, csplit, _ = pw.capi.gemm_last_config()
    return C, (plan, splits, csplit)


def _require_stream_k(cfg, plan):
    if cfg != (plan, 0, 1):
        pytest.skip(f"stream-K does not apply to plan {plan} on this device: {cfg}")


@pytest.mark.parametrize("plan", sorted(CASES))
def test_stream_k_matches_the_oracle(pw, plan):
    M, N, K = CASES[plan]
    assert pw.capi.gemm_bf16_set_plan(plan) == 0
    A = matrix_bf16(1300 + plan, M, K)
    B = matrix_bf16(1310 + plan, N, K)
    c0bits = matrix_bf16(1320 + plan, M, N)
    c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(torch.bfloat16)
    C, cfg = _launch(pw, A, B, M, N, K, torch.bfloat16, 0.5, 1.0, c0)
    _require_stream_k(cfg, plan)
    rows = sample_rows(M, seed=plan)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits, alpha=0.5, beta=1.0, rows=rows)
    rep = check(values_f64(C[torch.as_tensor(rows, device="cuda")]), Cref, R, out_bf16=True)
    assert rep["ok"], rep
    C2, _ = _launch(pw, A, B, M, N, K, torch.bfloat16, 0.5, 1.0, c0)
    assert torch.equal(C, C2)  # the fixup adds the parts in a fixed order


@pytest.mark.parametrize("plan", [4, 0])
def test_stream_k_integer_sums_bit_exact(pw, plan):
    """Small integers: every partial sum is exact in fp32, so the result is the oracle's bit for
    bit, in fp32 and after its one bf16 rounding."""
    M, N, K = CASES[plan]
    assert pw.capi.gemm_bf16_set_plan(plan) == 0
    rng = np.random.default_rng(1400 + plan)
    A = f64_to_bf16_bits(rng.integers(-2, 3, (M, K)).astype(np.float64))
    B = f64_to_bf16_bits(rng.integers(-2, 3, (N, K)).astype(np.float64))
    rows = sample_rows(M, seed=99)
    Cref, _ = oracle.gemm(A, B, M=M, N=N, K=K, rows=rows)
    idx = torch.as_tensor(rows, device="cuda")
    C, cfg = _launch(pw, A, B, M, N, K, torch.float32, 1.0, 0.0)
    _require_stream_k(cfg, plan)
    assert np.array_equal(values_f64(C[idx]), Cref)
    C, _ = _launch(pw, A, B, M, N, K, torch.bfloat16, 1.0, 0.0)
    assert np.array_equal(bits_of(C[idx]), f64_to_bf16_bits(Cref))


def test_stream_k_is_refused_where_it_does_not_apply(pw):
    """One wave or less: the forced switch falls back to the plain walk (no stream-K launch)."""
    assert pw.capi.gemm_bf16_set_plan(4) == 0
    M, N, K = 512, 1024, 2048  # 4 tiles
    A, B = matrix_bf16(1500, M, K), matrix_bf16(1501, N, K)
    C, cfg = _launch(pw, A, B, M, N, K, torch.float32, 1.0, 0.0)
    assert cfg[1] != 0
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, rows=sample_rows(M, seed=5))
    rep = check(values_f64(C[torch.as_tensor(sample_rows(M, seed=5), device="cuda")]), Cref, R, out_bf16=False)
    assert rep["ok"], rep


@pytest.mark.parametrize("plan", [4, 2])
def test_stream_k_batched_shared_w(pw, plan):
    """Stream-K on the batched shared-W call (MN-major X), alpha/beta with Y in place."""
    batch, M, K = 8, 1000, 2048
    N = 2048 if plan == 4 else 1024  # 128 tiles either way: more than the 74 CTA pairs
    assert pw.capi.gemm_bf16_set_plan(plan) == 0
    W = matrix_bf16(1600 + plan, M, K, std=K ** -0.5)
    X = matrix_bf16(1610 + plan, batch * K, N)
    y0 = torch.randn(batch, M, N, dtype=torch.float32, generator=torch.Generator().manual_seed(plan))
    y0 = y0.to(torch.bfloat16)
    Y = y0.clone().cuda()
    pw.gemm_bf16_batched_shared_w(to_dev_bf16(W), to_dev_bf16(X).view(batch, K, N), Y, alpha=0.5, beta=1.0)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    _require_stream_k(pw.capi.gemm_last_config()[:3], plan)
    rows = sample_rows(M, seed=plan)
    Cref, R = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * N,
                                  y0=y0.to(torch.float32).numpy().reshape(batch * M, N), stride_y=M * N,
                                  alpha=0.5, beta=1.0, rows=rows)
    got = values_f64(Y[:, torch.as_tensor(rows, device="cuda")])
    rep = check(got, Cref, R, out_bf16=True)
    assert rep["ok"], rep


def test_stream_k_fp16_operands_fp32_out(pw):
    """fp16 operands and fp32 output (the two-sub-tile plan's chunk-by-chunk epilogue)."""
    M, N, K = CASES[4]
    assert pw.capi.gemm_bf16_set_plan(4) == 0
    A, B = matrix_f16(1700, M, K), matrix_f16(1701, N, K)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    pw.gemm_bf16(to_dev_f16(A), to_dev_f16(B), C)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    _require_stream_k(pw.capi.gemm_last_config()[:3], 4)
    rows = sample_rows(M, seed=17)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, rows=rows, in_dtype="f16")
    rep = check(values_f64(C[torch.as_tensor(rows, device="cuda")]), Cref, R, out_bf16=False)
    assert rep["ok"], rep
