"""GPU parity of the persistent tcgen05 GEMM against the fp64 oracle, through the C ABI.

Every call goes through dsl_persistent_warp_b200 (ctypes -> libgemm_bf16.so).  Inputs are the
seeded synthetic matrices of synth/; expected values come only from oracle/.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import bits_of, check, sample_rows, to_dev_bf16, to_dev_f16, values_f64
from synth import (bf16_bits_to_f64, f16_bits_to_f64, f64_to_bf16_bits, f64_to_f16_bits, matrix_bf16,
                   matrix_f16, seed_for)

pytestmark = pytest.mark.gpu

PLANS = [0, 1, 2, 3, 4, 5, 6, 7, 8]


@pytest.fixture(scope="module")
def pw():
    import dsl_persistent_warp_b200 as m
    yield m
    m.capi.gemm_bf16_set_plan(-1)


def _plan(pw, plan):
    assert pw.capi.gemm_bf16_set_plan(plan) == 0


GUARD_ROWS = 3


def _run(pw, A, B, M, N, K, *, out=torch.bfloat16, alpha=1.0, beta=0.0, c0=None, ldc=None, f16=False):
    """A: (M, lda) uint16 bits, B: (N, ldb) bits (bf16, or fp16 with ``f16``).  C lives in a
    buffer with GUARD_ROWS extra NaN rows after row M-1; returns (C device view, buffer rows
    0..M-1); the guard rows are checked to be untouched here."""
    dev = to_dev_f16 if f16 else to_dev_bf16
    dA = dev(A)[:, :K]
    dB = dev(B)[:, :K]
    ldc = N if ldc is None else ldc
    full = torch.full((M + GUARD_ROWS, ldc), float("nan"), dtype=out, device="cuda")
    if c0 is not None:
        full[:M].copy_(c0.cuda())
    buf = full[:M]
    C = buf[:, :N]
    pw.gemm_bf16(dA, dB, C, alpha=alpha, beta=beta)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    assert torch.isnan(full[M:]).all().item(), "rows after C were written"
    return C, buf


# ----------------------------------------------------------------------------- exactness
@pytest.mark.parametrize("plan", PLANS)
def test_integer_inputs_bit_exact(pw, plan):
    """Small-integer inputs: every partial sum is an exact integer in fp32, so the GPU result
    must equal the oracle bit for bit (fp32 out), and its single bf16 rounding (bf16 out)."""
    _plan(pw, plan)
    rng = np.random.default_rng(100 + plan)
    M, N, K = 512, 384, 704
    Ai = rng.integers(-2, 3, (M, K)).astype(np.float64)
    Bi = rng.integers(-2, 3, (N, K)).astype(np.float64)
    A, B = f64_to_bf16_bits(Ai), f64_to_bf16_bits(Bi)
    Cref, _ = oracle.gemm(A, B, M=M, N=N, K=K)
    C, _ = _run(pw, A, B, M, N, K, out=torch.float32)
    assert np.array_equal(values_f64(C), Cref)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16)
    assert np.array_equal(bits_of(C), f64_to_bf16_bits(Cref))


@pytest.mark.parametrize("plan", PLANS)
def test_identity_and_permutation(pw, plan):
    """A = I reproduces B^T exactly; a permutation permutes rows exactly."""
    _plan(pw, plan)
    n = 320
    p = np.random.default_rng(7).permutation(n)
    P = np.zeros((n, n))
    P[np.arange(n), p] = 1.0
    B = matrix_bf16(77, 200, n)
    C, _ = _run(pw, f64_to_bf16_bits(P), B, n, 200, n, out=torch.float32)
    assert np.array_equal(values_f64(C), bf16_bits_to_f64(B).T[p, :])


# ----------------------------------------------------------------------------- config 1
@pytest.mark.parametrize("plan", PLANS)
def test_square_256_uniform_fp32(pw, plan):
    """M=N=K=256, U[-1,1] inputs, fp32 output, alpha=1, beta=0."""
    _plan(pw, plan)
    M = N = K = 256
    A = matrix_bf16(seed_for(0, "A"), M, K, dist="uniform")
    B = matrix_bf16(seed_for(0, "B"), N, K, dist="uniform")
    C, _ = _run(pw, A, B, M, N, K, out=torch.float32)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K)
    rep = check(values_f64(C), Cref, R, out_bf16=False)
    assert rep["ok"], rep


# ----------------------------------------------------------------------------- tails / edges
TAIL_SHAPES = [(1, 1, 1), (1, 8, 1), (3, 5, 7), (129, 257, 65), (300, 200, 100), (127, 129, 1000),
               (513, 264, 72), (64, 1000, 40), (1000, 16, 130)]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("shape", TAIL_SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in TAIL_SHAPES])
def test_ragged_shapes(pw, plan, shape):
    """Tile tails in M, N and K (TMA zero fill, clipped stores), bf16 and fp32 outputs, with
    alpha/beta and C read in place."""
    _plan(pw, plan)
    M, N, K = shape
    A = matrix_bf16(11, M, K, ld=K + (8 - K % 8) % 8)
    B = matrix_bf16(12, N, K, ld=K + (8 - K % 8) % 8)
    for out in (torch.float32, torch.bfloat16):
        ldc = N + (8 - N % 8) % 8 + 8
        c0bits = matrix_bf16(13, M, N, ld=ldc)
        c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(out)
        C, buf = _run(pw, A, B, M, N, K, out=out, alpha=0.5, beta=1.0, c0=c0, ldc=ldc)
        c0_np = c0[:, :N].to(torch.float32).numpy()
        Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0_np, alpha=0.5, beta=1.0)
        rep = check(values_f64(C), Cref, R, out_bf16=out == torch.bfloat16)
        assert rep["ok"], (out, rep)
        # the ldc padding columns keep their canary values
        pad_before = c0[:, N:].to(torch.float32).numpy()
        pad_after = buf[:, N:].cpu().to(torch.float32).numpy()
        assert np.array_equal(np.isnan(pad_before), np.isnan(pad_after))
        assert np.array_equal(pad_before[~np.isnan(pad_before)], pad_after[~np.isnan(pad_after)])


def test_beta_zero_ignores_nan_c(pw):
    _plan(pw, -1)
    M, N, K = 200, 136, 96
    A = matrix_bf16(21, M, K)
    B = matrix_bf16(22, N, K)
    C, _ = _run(pw, A, B, M, N, K, out=torch.float32)  # C starts as NaN
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K)
    assert check(values_f64(C), Cref, R, out_bf16=False)["ok"]


def test_k_zero_and_alpha_zero(pw):
    _plan(pw, -1)
    M, N = 70, 90
    c0 = torch.randn(M, N, dtype=torch.float32)
    C = c0.clone().cuda()
    A = torch.empty((M, 0), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((N, 0), dtype=torch.bfloat16, device="cuda")
    pw.gemm_bf16(A, B, C, alpha=1.0, beta=-2.0)
    torch.cuda.synchronize()
    assert torch.equal(C.cpu(), -2.0 * c0)
    Ab = to_dev_bf16(matrix_bf16(1, M, 64))
    Bb = to_dev_bf16(matrix_bf16(2, N, 64))
    C = torch.full((M, N), float("nan"), device="cuda")
    pw.gemm_bf16(Ab, Bb, C, alpha=0.0, beta=0.0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(C).item() == 0


def test_unaligned_leading_dimensions(pw):
    """lda/ldb not a multiple of 8 (pre-pass copy) and ldc odd (direct-store epilogue)."""
    _plan(pw, -1)
    M, N, K = 261, 133, 203
    A = matrix_bf16(31, M, K, ld=K)  # lda = 203: not TMA-able
    B = matrix_bf16(32, N, K, ld=K + 2)
    ldc = N  # 133: odd
    c0bits = matrix_bf16(33, M, N, ld=ldc)
    c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(torch.bfloat16)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0, ldc=ldc)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits, alpha=0.5, beta=1.0)
    rep = check(values_f64(C), Cref, R, out_bf16=True)
    assert rep["ok"], rep


def test_misaligned_base_pointer(pw):
    """A base that is 2-byte but not 16-byte aligned goes through the pre-pass copy."""
    _plan(pw, -1)
    M, N, K = 150, 140, 128
    Abits = matrix_bf16(41, M * K + 1, 1).reshape(-1)
    Bbits = matrix_bf16(42, N, K)
    dA_full = to_dev_bf16(Abits)
    dA = dA_full[1:].view(M, K)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    pw.gemm_bf16(dA, to_dev_bf16(Bbits), C)
    torch.cuda.synchronize()
    Cref, R = oracle.gemm(Abits[1:].reshape(M, K), Bbits, M=M, N=N, K=K)
    assert check(values_f64(C), Cref, R, out_bf16=False)["ok"]


@pytest.mark.parametrize("plan", PLANS)
def test_deterministic(pw, plan):
    _plan(pw, plan)
    M, N, K = 700, 900, 1100
    A = to_dev_bf16(matrix_bf16(51, M, K))
    B = to_dev_bf16(matrix_bf16(52, N, K))
    C1 = pw.gemm_bf16(A, B, out_dtype=torch.float32)
    C2 = pw.gemm_bf16(A, B, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(C1, C2)


# ----------------------------------------------------------------------------- split-K
# (M, N, K, slices): every slice count divides the k-blocks (BK = 64) into equal runs but the
# last, and the K tail (K % 64 != 0) lands in the last slice.
SPLIT_CASES = [(300, 200, 1100, 2), (129, 257, 1500, 3), (1000, 136, 2000, 5), (256, 512, 1024, 8)]
STREAM_PLANS = [0, 1, 2, 3, 4, 8]


@pytest.mark.parametrize("plan", STREAM_PLANS)
@pytest.mark.parametrize("case", SPLIT_CASES, ids=[f"{m}x{n}x{k}_s{s}" for m, n, k, s in SPLIT_CASES])
def test_split_k(pw, plan, case, monkeypatch):
    """K cut into slices whose fp32 partial sums the last-arriving unit adds in slice order:
    same tolerance as the unsplit path, C read in place with alpha/beta, ragged M and N."""
    M, N, K, S = case
    monkeypatch.setenv("GEMM_BF16_SPLIT_K", str(S))
    _plan(pw, plan)
    A = matrix_bf16(61, M, K)
    B = matrix_bf16(62, N, K)
    c0bits = matrix_bf16(63, M, N)
    c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(torch.bfloat16)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits, alpha=0.5, beta=1.0)
    rep = check(values_f64(C), Cref, R, out_bf16=True)
    assert rep["ok"], rep
    # the same call again gives the same bits whatever order the slices arrived in
    C2, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0)
    assert torch.equal(C, C2)


@pytest.mark.parametrize("plan", STREAM_PLANS)
def test_split_k_integer_bit_exact(pw, plan, monkeypatch):
    """Small-integer inputs: slice sums and their total are exact in fp32, so a split GEMM must
    match the oracle bit for bit."""
    monkeypatch.setenv("GEMM_BF16_SPLIT_K", "4")
    _plan(pw, plan)
    rng = np.random.default_rng(200 + plan)
    M, N, K = 384, 272, 2048
    A = f64_to_bf16_bits(rng.integers(-3, 4, (M, K)).astype(np.float64))
    B = f64_to_bf16_bits(rng.integers(-3, 4, (N, K)).astype(np.float64))
    Cref, _ = oracle.gemm(A, B, M=M, N=N, K=K)
    C, _ = _run(pw, A, B, M, N, K, out=torch.float32)
    assert np.array_equal(values_f64(C), Cref)


def test_split_k_unaligned_c(pw, monkeypatch):
    """Split-K with an odd ldc: the fixup goes out through the row-by-row coalesced store."""
    monkeypatch.setenv("GEMM_BF16_SPLIT_K", "2")
    _plan(pw, -1)
    M, N, K = 261, 133, 1203
    A = matrix_bf16(71, M, K, ld=K)
    B = matrix_bf16(72, N, K, ld=K + 2)
    c0bits = matrix_bf16(73, M, N, ld=N)
    c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(torch.bfloat16)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0, ldc=N)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits, alpha=0.5, beta=1.0)
    rep = check(values_f64(C), Cref, R, out_bf16=True)
    assert rep["ok"], rep


# ----------------------------------------------------------------------------- cluster split-K
# Streaming plans with one MMA sub-tile: the ones whose kernels take it.  The 2-CTA plans (2, 3)
# cut K over CTA pairs, so at most 4 slices fit a cluster of 8.
CSPLIT_PLANS = [0, 1, 8, 2, 3]
CG2_PLANS = (2, 3)


def _csplit_fits(plan, S):
    return S * (2 if plan in CG2_PLANS else 1) <= 8
CSPLIT_CASES = [(300, 200, 1100, 2), (129, 257, 1500, 4), (1000, 136, 2000, 8), (256, 512, 1024, 4),
                (127, 1000, 2048, 4)]


@pytest.mark.parametrize("plan", CSPLIT_PLANS)
@pytest.mark.parametrize("case", CSPLIT_CASES, ids=[f"{m}x{n}x{k}_c{s}" for m, n, k, s in CSPLIT_CASES])
def test_cluster_split_k(pw, plan, case, monkeypatch):
    """K slices of a tile on the CTAs of one cluster, partial tiles added through distributed
    shared memory: same tolerance as the unsplit path, alpha/beta with C in place, ragged M, N
    and K; a second call gives the same bits."""
    M, N, K, S = case
    if not _csplit_fits(plan, S):
        S //= 2
    monkeypatch.setenv("GEMM_BF16_CLUSTER_SPLIT", str(S))
    _plan(pw, plan)
    A = matrix_bf16(161, M, K)
    B = matrix_bf16(162, N, K)
    c0bits = matrix_bf16(163, M, N)
    c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(torch.bfloat16)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits, alpha=0.5, beta=1.0)
    rep = check(values_f64(C), Cref, R, out_bf16=True)
    assert rep["ok"], rep
    C2, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0)
    assert torch.equal(C, C2)


@pytest.mark.parametrize("plan", CSPLIT_PLANS)
@pytest.mark.parametrize("S", [2, 4, 8])
def test_cluster_split_k_integer_bit_exact(pw, plan, S, monkeypatch):
    """Small-integer inputs: the slice sums and their total are exact in fp32, so the result is
    bit-exact against the oracle, in fp32 and in bf16."""
    if not _csplit_fits(plan, S):
        pytest.skip("a cluster of CTA pairs holds at most 4 slices")
    monkeypatch.setenv("GEMM_BF16_CLUSTER_SPLIT", str(S))
    _plan(pw, plan)
    rng = np.random.default_rng(700 + plan + S)
    M, N, K = 384, 272, 2048
    A = f64_to_bf16_bits(rng.integers(-3, 4, (M, K)).astype(np.float64))
    B = f64_to_bf16_bits(rng.integers(-3, 4, (N, K)).astype(np.float64))
    Cref, _ = oracle.gemm(A, B, M=M, N=N, K=K)
    C, _ = _run(pw, A, B, M, N, K, out=torch.float32)
    assert np.array_equal(values_f64(C), Cref)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16)
    assert np.array_equal(bits_of(C), f64_to_bf16_bits(Cref))


def test_cluster_split_k_unaligned_c_and_fp16(pw, monkeypatch):
    """Cluster split-K with an odd ldc (row-by-row epilogue) and packed lda/ldb (pre-pass), and
    with fp16 operands and fp16 output."""
    monkeypatch.setenv("GEMM_BF16_CLUSTER_SPLIT", "4")
    _plan(pw, -1)
    M, N, K = 127, 8191, 2048
    A = matrix_bf16(171, M, K, ld=K)
    B = matrix_bf16(172, N, K, ld=K)
    c0bits = matrix_bf16(173, M, N, ld=N)
    c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(torch.bfloat16)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0, ldc=N)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits, alpha=0.5, beta=1.0)
    rep = check(values_f64(C), Cref, R, out_bf16=True)
    assert rep["ok"], rep
    M, N, K = 300, 520, 3000
    A = matrix_f16(174, M, K)
    B = matrix_f16(175, N, K)
    C, _ = _run(pw, A, B, M, N, K, out=torch.float16, f16=True)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, in_dtype="f16")
    rep = check(values_f64(C), Cref, R, out_bf16=False, out_f16=True)
    assert rep["ok"], rep


@pytest.mark.parametrize("plan", CSPLIT_PLANS)
def test_batched_cluster_split_k(pw, plan, monkeypatch):
    """Cluster split-K on the batched shared-W call (MN-major X)."""
    monkeypatch.setenv("GEMM_BF16_CLUSTER_SPLIT", "2")
    _plan(pw, plan)
    batch, M, N, K = 3, 200, 128, 2048
    W = matrix_bf16(181, M, K, std=K ** -0.5)
    X = matrix_bf16(182, batch * K, N)
    y0 = torch.randn(batch, M, N, dtype=torch.float32).to(torch.bfloat16)
    Y = y0.clone().cuda()
    pw.gemm_bf16_batched_shared_w(to_dev_bf16(W), to_dev_bf16(X).view(batch, K, N), Y, alpha=0.5, beta=1.0)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    Cref, R = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * N,
                                  y0=y0.to(torch.float32).numpy().reshape(batch * M, N), stride_y=M * N,
                                  alpha=0.5, beta=1.0)
    rep = check(values_f64(Y), Cref, R, out_bf16=True)
    assert rep["ok"], rep


def test_abi_errors_on_gpu(pw):
    c = pw.capi
    t = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    assert c.gemm_bf16(4, 4, 4, p, 3, p, 4, p, 4, 1, 1.0, 0.0, s) == c.GEMM_ERR_INVALID_ARG
    assert c.gemm_bf16(4, 4, 4, p, 4, p, 4, p, 4, 7, 1.0, 0.0, s) == c.GEMM_ERR_INVALID_ARG
    assert c.gemm_bf16(4, 4, 4, p + 1, 4, p, 4, p, 4, 1, 1.0, 0.0, s) == c.GEMM_ERR_INVALID_ARG
    assert c.gemm_bf16(4, 4, 4, None, 4, p, 4, p, 4, 1, 1.0, 0.0, s) == c.GEMM_ERR_INVALID_ARG
    assert c.gemm_bf16(4, 4, 4, p, 4, p, 4, p + 2, 4, 0, 1.0, 0.0, s) == c.GEMM_ERR_INVALID_ARG
    assert c.gemm_bf16(0, 4, 4, None, 4, None, 4, None, 4, 1, 1.0, 0.0, s) == c.GEMM_OK
    torch.cuda.synchronize()


# ----------------------------------------------------------------------------- batched
# (batch, M, N, K).  N = 64, 128 or 256 lets wide tiles hold several batch entries side by side
# (with an odd batch count the last tile is partly empty); N = 72 and 264 cannot be packed.
BATCH_CASES = [(3, 256, 128, 512), (5, 100, 72, 200), (2, 300, 264, 130), (64, 256, 128, 512),
               (5, 256, 64, 256), (7, 128, 128, 512), (3, 200, 256, 320)]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("case", BATCH_CASES, ids=[f"b{b}_{m}x{n}x{k}" for b, m, n, k in BATCH_CASES])
def test_batched_shared_w(pw, plan, case):
    _plan(pw, plan)
    batch, M, N, K = case
    ldx = N + (8 - N % 8) % 8
    W = matrix_bf16(61, M, K, std=512 ** -0.5)
    X = matrix_bf16(62, batch * K, N, ld=ldx)
    for out, beta in ((torch.bfloat16, 0.0), (torch.float32, 1.0)):
        dW = to_dev_bf16(W)
        dX = to_dev_bf16(X).view(batch, K, ldx)[:, :, :N]
        y0 = torch.randn(batch, M, N, dtype=torch.float32).to(out)
        Y = y0.clone().cuda()
        pw.gemm_bf16_batched_shared_w(dW, dX, Y, alpha=1.0, beta=beta)
        torch.cuda.synchronize()
        assert pw.device_status() == 0
        Cref, R = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * ldx,
                                      y0=y0.to(torch.float32).numpy().reshape(batch * M, N),
                                      stride_y=M * N, alpha=1.0, beta=beta)
        rep = check(values_f64(Y), Cref, R, out_bf16=out == torch.bfloat16)
        assert rep["ok"], (out, rep)


# (batch, M, N, K, slices): N = 128 and 64 are packed several entries to a wide tile by
# plans 1, 2 and 4; the others take one entry per tile.
SPLIT_BATCH_CASES = [(3, 256, 128, 1024, 2), (5, 100, 72, 1100, 3), (4, 128, 64, 2048, 4)]


@pytest.mark.parametrize("plan", STREAM_PLANS)
@pytest.mark.parametrize("case", SPLIT_BATCH_CASES,
                         ids=[f"b{b}_{m}x{n}x{k}_s{s}" for b, m, n, k, s in SPLIT_BATCH_CASES])
def test_batched_split_k(pw, plan, case, monkeypatch):
    """Split-K on the batched shared-W call: tiles over (b, n) with MN-major X, packing included."""
    batch, M, N, K, S = case
    monkeypatch.setenv("GEMM_BF16_SPLIT_K", str(S))
    _plan(pw, plan)
    ldx = N + (8 - N % 8) % 8
    W = matrix_bf16(81, M, K, std=K ** -0.5)
    X = matrix_bf16(82, batch * K, N, ld=ldx)
    dW = to_dev_bf16(W)
    dX = to_dev_bf16(X).view(batch, K, ldx)[:, :, :N]
    y0 = torch.randn(batch, M, N, dtype=torch.float32).to(torch.bfloat16)
    Y = y0.clone().cuda()
    pw.gemm_bf16_batched_shared_w(dW, dX, Y, alpha=0.5, beta=1.0)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    Cref, R = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * ldx,
                                  y0=y0.to(torch.float32).numpy().reshape(batch * M, N),
                                  stride_y=M * N, alpha=0.5, beta=1.0)
    rep = check(values_f64(Y), Cref, R, out_bf16=True)
    assert rep["ok"], rep


# ----------------------------------------------------------------------------- full configs
def _full_case(pw, idx, M, N, K, *, std_a=1.0, std_b=1.0, alpha=1.0, beta=0.0, rows=None):
    _plan(pw, -1)
    A = matrix_bf16(seed_for(idx, "A"), M, K, std=std_a)
    B = matrix_bf16(seed_for(idx, "B"), N, K, std=std_b)
    c0 = None
    if beta != 0.0:
        c0bits = matrix_bf16(seed_for(idx, "C"), M, N)
        c0 = torch.from_numpy(c0bits.view(np.int16)).view(torch.bfloat16)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=alpha, beta=beta, c0=c0)
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=None if c0 is None else c0bits, alpha=alpha,
                          beta=beta, rows=rows)
    Cg = values_f64(C if rows is None else C[torch.as_tensor(rows, device="cuda")])
    rep = check(Cg, Cref, R, out_bf16=True)
    assert rep["ok"], rep
    return C, A, B


@pytest.mark.parametrize("n", [4096, 8192])
def test_square_bf16(pw, n):
    """M=N=K=4096 and 8192, N(0,1) inputs, bf16 output: sampled rows vs the oracle (every
    output tile, both tile borders)."""
    _full_case(pw, 1, n, n, n, rows=sample_rows(n, seed=n))


@pytest.mark.parametrize("which", ["up", "down"])
def test_llm_mlp_shapes(pw, which):
    """LLM MLP GEMMs: up-proj 16384x28672x8192 and down-proj 16384x8192x28672, activations
    N(0,1), weights N(0,0.02), bf16 out: sampled rows vs the oracle."""
    M, N, K = (16384, 28672, 8192) if which == "up" else (16384, 8192, 28672)
    _full_case(pw, 2, M, N, K, std_b=0.02, rows=sample_rows(M, seed=K))


EDGE = [(4099, 4099, 4099), (8192, 256, 4096), (127, 8191, 2048)]


@pytest.mark.parametrize("shape", EDGE, ids=[f"{m}x{n}x{k}" for m, n, k in EDGE])
def test_edge_shapes(pw, shape):
    """Edge shapes with alpha=0.5, beta=1 and C ~ N(0,1) bf16 in place (packed leading
    dimensions, so 4099 and 8191 take the alignment pre-pass / direct-store paths)."""
    M, N, K = shape
    rows = None if M * N * K <= 8192 * 256 * 4096 else sample_rows(M, seed=M)
    _full_case(pw, 3, M, N, K, alpha=0.5, beta=1.0, rows=rows)


# Few output tiles and a long K: the planner cuts K into slices on its own here.
DEEP_K = [(1024, 1024, 8192), (512, 512, 16384), (384, 1000, 8192)]


@pytest.mark.parametrize("shape", DEEP_K, ids=[f"{m}x{n}x{k}" for m, n, k in DEEP_K])
def test_deep_k_auto_split(pw, shape):
    """Automatic plan and split-K choice on deep-K shapes, alpha/beta with C in place, against
    the oracle on every row; a second call must give the same bits."""
    M, N, K = shape
    C, A, B = _full_case(pw, 7, M, N, K, std_a=K ** -0.5, alpha=0.5, beta=1.0)
    c0bits = matrix_bf16(seed_for(7, "C"), M, N)
    c0 = torch.from_numpy(c0bits.view(np.int16)).view(torch.bfloat16)
    C2, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, alpha=0.5, beta=1.0, c0=c0)
    assert torch.equal(C, C2)


def test_recsys_batched_config(pw):
    """Y[b] = W X[b], b < 2048, W 256x512 ~ N(0, 1/sqrt(512)), X[b] 512x128 ~ N(0,1), bf16 out.
    All batches on sampled rows, and 16 whole batches."""
    _plan(pw, -1)
    batch, M, K, N = 2048, 256, 512, 128
    W = matrix_bf16(seed_for(4, "W"), M, K, std=512 ** -0.5)
    X = matrix_bf16(seed_for(4, "X"), batch * K, N)
    dW, dX = to_dev_bf16(W), to_dev_bf16(X).view(batch, K, N)
    Y = pw.gemm_bf16_batched_shared_w(dW, dX)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    rows = [0, 1, 77, 127, 128, 200, 255]
    Cref, R = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * N, rows=rows)
    Yv = values_f64(Y[:, rows, :])
    rep = check(Yv, Cref, R, out_bf16=True)
    assert rep["ok"], rep
    sel = np.random.default_rng(4).choice(batch, 16, replace=False)
    for b in sel:
        Cb, Rb = oracle.gemm(W, X[b * K:(b + 1) * K], M=M, N=N, K=K, b_kmajor=False)
        rep = check(values_f64(Y[int(b)]), Cb, Rb, out_bf16=True)
        assert rep["ok"], (int(b), rep)


# ----------------------------------------------------------------------------- bit-exact at size
def test_edge4099_integer_bit_exact(pw):
    """M = N = K = 4099 with packed leading dimensions (alignment pre-pass for A and B, the
    row-by-row epilogue for C), alpha = 0.5, beta = 1, small-integer A, B and C: every partial
    sum and alpha*acc + beta*c0 are exact in fp32, so the fp32 output equals the oracle bit for
    bit and the bf16 output is its single round-to-nearest-even."""
    _plan(pw, -1)
    n = 4099
    rng = np.random.default_rng(4099)
    A = f64_to_bf16_bits(rng.integers(-2, 3, (n, n)).astype(np.float64))
    B = f64_to_bf16_bits(rng.integers(-2, 3, (n, n)).astype(np.float64))
    c0i = rng.integers(-2, 3, (n, n)).astype(np.float64)
    Cref, _ = oracle.gemm(A, B, M=n, N=n, K=n, c0=c0i.astype(np.float32), alpha=0.5, beta=1.0)
    C, _ = _run(pw, A, B, n, n, n, out=torch.float32, alpha=0.5, beta=1.0,
                c0=torch.from_numpy(c0i.astype(np.float32)))
    assert np.array_equal(values_f64(C), Cref)
    C, _ = _run(pw, A, B, n, n, n, out=torch.bfloat16, alpha=0.5, beta=1.0,
                c0=torch.from_numpy(c0i).to(torch.bfloat16))
    assert np.array_equal(bits_of(C), f64_to_bf16_bits(Cref))


BATCH_EXACT = [(6, 256, 128, 512), (3, 200, 264, 320)]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("case", BATCH_EXACT, ids=[f"b{b}_{m}x{n}x{k}" for b, m, n, k in BATCH_EXACT])
def test_batched_integer_bit_exact(pw, plan, case):
    """Shared-W batches (MN-major X descriptors, packing for N = 128) with small-integer
    inputs: bit-exact against the oracle in fp32 and in bf16."""
    _plan(pw, plan)
    batch, M, N, K = case
    rng = np.random.default_rng(300 + plan)
    W = f64_to_bf16_bits(rng.integers(-3, 4, (M, K)).astype(np.float64))
    X = f64_to_bf16_bits(rng.integers(-3, 4, (batch * K, N)).astype(np.float64))
    Cref, _ = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * N)
    dW, dX = to_dev_bf16(W), to_dev_bf16(X).view(batch, K, N)
    for out in (torch.float32, torch.bfloat16):
        Y = pw.gemm_bf16_batched_shared_w(dW, dX, out_dtype=out)
        torch.cuda.synchronize()
        assert pw.device_status() == 0
        if out == torch.float32:
            assert np.array_equal(values_f64(Y), Cref)
        else:
            assert np.array_equal(bits_of(Y), f64_to_bf16_bits(Cref))


# ----------------------------------------------------------------------------- fp16 operands
@pytest.mark.parametrize("plan", PLANS)
def test_f16_integer_bit_exact(pw, plan):
    """fp16 operands: A holds integers up to +-1000 (exact in fp16, not in bf16), B holds
    -1, 0, 1; every partial sum is an exact integer below 2^24, so the fp32 output equals the
    oracle bit for bit, and an fp16 output is its single rounding."""
    _plan(pw, plan)
    rng = np.random.default_rng(500 + plan)
    M, N, K = 512, 384, 704
    A = f64_to_f16_bits(rng.integers(-1000, 1001, (M, K)).astype(np.float64))
    B = f64_to_f16_bits(rng.integers(-1, 2, (N, K)).astype(np.float64))
    Cref, _ = oracle.gemm(A, B, M=M, N=N, K=K, in_dtype="f16")
    C, _ = _run(pw, A, B, M, N, K, out=torch.float32, f16=True)
    assert np.array_equal(values_f64(C), Cref)
    C, _ = _run(pw, A, B, M, N, K, out=torch.bfloat16, f16=True)
    assert np.array_equal(bits_of(C), f64_to_bf16_bits(Cref))


F16_SHAPES = [(129, 257, 65), (300, 200, 1100), (513, 264, 72), (1000, 16, 130)]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("shape", F16_SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in F16_SHAPES])
def test_f16_ragged(pw, plan, shape):
    """fp16 operands (values down to the subnormal range) and every output type, with
    alpha/beta and C read in place, ragged M, N and K."""
    _plan(pw, plan)
    M, N, K = shape
    A = matrix_f16(111, M, K, std=0.05, ld=K + (8 - K % 8) % 8)
    B = matrix_f16(112, N, K, ld=K + (8 - K % 8) % 8)
    for out in (torch.float16, torch.float32, torch.bfloat16):
        ldc = N + (8 - N % 8) % 8 + 8
        c0 = torch.from_numpy(f16_bits_to_f64(matrix_f16(113, M, N, ld=ldc))).to(out)
        C, buf = _run(pw, A, B, M, N, K, out=out, alpha=0.5, beta=1.0, c0=c0, ldc=ldc, f16=True)
        c0_np = c0[:, :N].to(torch.float32).numpy()
        Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0_np, alpha=0.5, beta=1.0, in_dtype="f16")
        rep = check(values_f64(C), Cref, R, out_bf16=out == torch.bfloat16, out_f16=out == torch.float16)
        assert rep["ok"], (out, rep)
        pad_before = c0[:, N:].to(torch.float32).numpy()
        pad_after = buf[:, N:].cpu().to(torch.float32).numpy()
        assert np.array_equal(np.isnan(pad_before), np.isnan(pad_after))


@pytest.mark.parametrize("plan", PLANS)
def test_f16_batched_shared_w(pw, plan):
    _plan(pw, plan)
    batch, M, N, K = 5, 256, 128, 512
    W = matrix_f16(121, M, K, std=512 ** -0.5)
    X = matrix_f16(122, batch * K, N)
    dW, dX = to_dev_f16(W), to_dev_f16(X).view(batch, K, N)
    for out in (torch.float16, torch.float32):
        Y = pw.gemm_bf16_batched_shared_w(dW, dX, out_dtype=out)
        torch.cuda.synchronize()
        assert pw.device_status() == 0
        Cref, R = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * N, in_dtype="f16")
        rep = check(values_f64(Y), Cref, R, out_bf16=False, out_f16=out == torch.float16)
        assert rep["ok"], (out, rep)


def test_f16_square8192(pw):
    """M = N = K = 8192 with fp16 operands N(0,1) and fp16 output: sampled rows vs the oracle."""
    _plan(pw, -1)
    n = 8192
    A = matrix_f16(seed_for(1, "A"), n, n)
    B = matrix_f16(seed_for(1, "B"), n, n)
    C, _ = _run(pw, A, B, n, n, n, out=torch.float16, f16=True)
    rows = sample_rows(n, seed=16)
    Cref, R = oracle.gemm(A, B, M=n, N=n, K=n, rows=rows, in_dtype="f16")
    rep = check(values_f64(C[torch.as_tensor(rows, device="cuda")]), Cref, R, out_bf16=False, out_f16=True)
    assert rep["ok"], rep


# ----------------------------------------------------------------------------- tensor-map cache
def test_tensor_map_cache_hits_on_repeated_calls(pw):
    """A second call on the same buffers encodes no tensor map: its three maps (A, B, C) come
    from the cache."""
    _plan(pw, -1)
    A = to_dev_bf16(matrix_bf16(131, 384, 256))
    B = to_dev_bf16(matrix_bf16(132, 320, 256))
    C = torch.empty((384, 320), dtype=torch.bfloat16, device="cuda")
    pw.gemm_bf16(A, B, C)
    h0, m0 = pw.capi.gemm_bf16_tensor_map_cache_stats()
    pw.gemm_bf16(A, B, C)
    torch.cuda.synchronize()
    h1, m1 = pw.capi.gemm_bf16_tensor_map_cache_stats()
    assert (h1 - h0, m1 - m0) == (3, 0)


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_large_unaligned_c(pw, out):
    """C that tensor stores cannot address (odd ldc; a base one element off a 16-byte boundary)
    on a multi-wave GEMM: the result, with beta = 0 and beta = 1, matches the oracle and the
    columns past N and the elements around C keep their canaries."""
    _plan(pw, -1)
    M, N, K = 2100, 2050, 320
    A = matrix_bf16(1801, M, K)
    B = matrix_bf16(1802, N, K)
    ldc = 2053
    c0bits = matrix_bf16(1803, M, N, ld=ldc)
    c0 = torch.from_numpy(bf16_bits_to_f64(c0bits)).to(out)
    for beta in (0.0, 1.0):
        C, buf = _run(pw, A, B, M, N, K, out=out, alpha=0.5, beta=beta, c0=c0, ldc=ldc)
        Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0bits if beta else None, alpha=0.5, beta=beta)
        rep = check(values_f64(C), Cref, R, out_bf16=out == torch.bfloat16)
        assert rep["ok"], (beta, rep)
        pad_before = c0[:, N:].to(torch.float32).numpy()
        pad_after = buf[:, N:].cpu().to(torch.float32).numpy()
        assert np.array_equal(np.isnan(pad_before), np.isnan(pad_after))
        assert np.array_equal(pad_before[~np.isnan(pad_before)], pad_after[~np.isnan(pad_after)])
    # aligned ldc, base one element past a 16-byte boundary
    ldc = 2056
    full = torch.full((M * ldc + 8,), float("nan"), dtype=out, device="cuda")
    C = full[1:1 + M * ldc].view(M, ldc)[:, :N]
    pw.gemm_bf16(to_dev_bf16(A), to_dev_bf16(B), C, alpha=0.5, beta=0.0)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, alpha=0.5)
    rep = check(values_f64(C), Cref, R, out_bf16=out == torch.bfloat16)
    assert rep["ok"], rep
    assert torch.isnan(full[0]).item() and torch.isnan(full[1 + M * ldc:]).all().item()
    assert torch.isnan(full[1:1 + M * ldc].view(M, ldc)[:, N:]).all().item()
