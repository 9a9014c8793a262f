"""GPU parity of the deduplicated shared-W form (gemm_bf16_batched_shared_w_dedup) against the
oracle's definition: every item b is its own GEMM Y[b] = alpha * W * X[index[b]] + beta * Y[b],
with X holding only the distinct entries.  Calls go through the C ABI (ctypes)."""
import numpy as np
import pytest
import torch

import oracle
from parity import bits_of, check, to_dev_bf16, values_f64
from synth import matrix_bf16, seed_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pw():
    import dsl_persistent_warp_b200 as m
    yield m
    m.capi.gemm_bf16_set_plan(-1)


def _index(kind, batch, n_unique, seed=0):
    if kind == "requests":  # consecutive items share one entry (items scored for one buyer)
        return (np.arange(batch) * n_unique // batch).astype(np.int32)
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, n_unique, batch).astype(np.int32)
    idx[idx == n_unique - 1] = 0  # leave the last entry unused
    return idx


# (batch, n_unique, M, N, K, index kind): N = 128 packs two entries per 256-wide tile; N = 72
# cannot be packed.
CASES = [(256, 2, 256, 128, 512, "requests"), (300, 37, 256, 128, 512, "random"),
         (64, 5, 200, 72, 320, "random"), (40, 40, 128, 64, 256, "requests"), (17, 1, 256, 128, 512, "requests")]


@pytest.mark.parametrize("case", CASES, ids=[f"b{b}_u{u}_{m}x{n}x{k}_{t}" for b, u, m, n, k, t in CASES])
def test_dedup_matches_the_oracle(pw, case):
    pw.capi.gemm_bf16_set_plan(-1)
    batch, n_u, M, N, K, kind = case
    index = _index(kind, batch, n_u, seed=batch)
    W = matrix_bf16(seed_for(4, "W"), M, K, std=K ** -0.5)
    X = matrix_bf16(seed_for(4, "X"), n_u * K, N)
    y0 = torch.randn(batch, M, N, dtype=torch.float32).to(torch.bfloat16)
    for out, beta in ((torch.bfloat16, 0.0), (torch.bfloat16, 1.0), (torch.float32, 0.0)):
        Y = y0.to(out).cuda()
        pw.gemm_bf16_batched_shared_w_dedup(to_dev_bf16(W), to_dev_bf16(X).view(n_u, K, N),
                                            torch.from_numpy(index).cuda(), Y, alpha=0.5, beta=beta)
        torch.cuda.synchronize()
        assert pw.device_status() == 0
        Cref, R = oracle.gemm_batched_dedup(W, X, index, n_x=n_u, M=M, N=N, K=K, stride_x=K * N,
                                            y0=y0.to(torch.float32).numpy().reshape(batch * M, N),
                                            stride_y=M * N, alpha=0.5, beta=beta)
        rep = check(values_f64(Y), Cref, R, out_bf16=out == torch.bfloat16)
        assert rep["ok"], (out, beta, rep)


@pytest.mark.parametrize("plan", [0, 2, 7, 8])
def test_dedup_bitwise_equals_the_expanded_batch(pw, plan):
    """The same tile plan on the expanded batch X[b] = X[index[b]] gives the same bits."""
    pw.capi.gemm_bf16_set_plan(plan)
    batch, n_u, M, N, K = 384, 3, 256, 128, 512
    index = _index("requests", batch, n_u)
    W = matrix_bf16(41, M, K, std=K ** -0.5)
    X = matrix_bf16(42, n_u * K, N)
    dX = to_dev_bf16(X).view(n_u, K, N)
    Yd = pw.gemm_bf16_batched_shared_w_dedup(to_dev_bf16(W), dX, torch.from_numpy(index).cuda())
    Xe = dX[torch.from_numpy(index).long().cuda()].contiguous()
    Ye = pw.gemm_bf16_batched_shared_w(to_dev_bf16(W), Xe)
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    assert np.array_equal(bits_of(Yd), bits_of(Ye))


def test_recsys_shape_with_requests_of_128(pw):
    """The RecSys shape (2048 items, W 256x512, X entries 512x128) with 16 requests of 128
    items each sharing one entry: sampled items and rows against the oracle."""
    pw.capi.gemm_bf16_set_plan(-1)
    batch, n_u, M, K, N = 2048, 16, 256, 512, 128
    index = _index("requests", batch, n_u)
    W = matrix_bf16(seed_for(4, "W"), M, K, std=512 ** -0.5)
    X = matrix_bf16(seed_for(4, "X"), n_u * K, N)
    Y = pw.gemm_bf16_batched_shared_w_dedup(to_dev_bf16(W), to_dev_bf16(X).view(n_u, K, N),
                                            torch.from_numpy(index).cuda())
    torch.cuda.synchronize()
    assert pw.device_status() == 0
    items = np.random.default_rng(5).choice(batch, 64, replace=False)
    rows = [0, 31, 32, 100, 127, 128, 200, 255]
    Cref, R = oracle.gemm_batched_dedup(W, X, index[items], n_x=n_u, M=M, N=N, K=K, stride_x=K * N, rows=rows)
    Yv = values_f64(Y[torch.as_tensor(items, device="cuda")][:, rows, :])
    rep = check(Yv, Cref, R, out_bf16=True)
    assert rep["ok"], rep


def test_dedup_index_out_of_range_is_reported(pw):
    """An index outside [0, n_unique) leaves that item's Y untouched, the others are computed,
    and the device status reports an invalid argument."""
    pw.capi.gemm_bf16_set_plan(-1)
    batch, n_u, M, N, K = 8, 2, 128, 64, 128
    index = np.array([0, 1, 1, 5, 0, -1, 1, 0], dtype=np.int32)
    W = matrix_bf16(51, M, K)
    X = matrix_bf16(52, n_u * K, N)
    Y = torch.full((batch, M, N), 3.0, dtype=torch.float32, device="cuda")
    pw.gemm_bf16_batched_shared_w_dedup(to_dev_bf16(W), to_dev_bf16(X).view(n_u, K, N),
                                        torch.from_numpy(index).cuda(), Y)
    assert pw.device_status() == pw.capi.GEMM_ERR_INVALID_ARG
    assert pw.device_status() == 0  # the status word was cleared
    Yc = Y.cpu()
    assert bool((Yc[3] == 3.0).all()) and bool((Yc[5] == 3.0).all())
    good = [0, 1, 2, 4, 6, 7]
    Cref, R = oracle.gemm_batched_dedup(W, X, index[good], n_x=n_u, M=M, N=N, K=K, stride_x=K * N)
    assert check(values_f64(Yc[good]), Cref, R, out_bf16=False)["ok"]
