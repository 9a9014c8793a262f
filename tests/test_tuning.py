"""The autotuner's table through the C ABI: save/load/clear on the CPU (no GPU), and on a B200
the tuner's measurements, the use of their result by later calls, and that it leaves C alone."""
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

GOOD = """# tuned on a B200 (148 SMs)
gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 1 1 4 8 31.250
gemmtune1 148 2048 256 128 512 0 1 0 1 0 1 1 1 7 1 1 8 80.500
gemmtune1 148 1 4096 4096 4096 0 0 0 1 0 1 1 1 4 0 1 16 95.000
"""


@pytest.fixture()
def capi():
    from conftest import build_library
    build_library()
    from dsl_persistent_warp_b200 import capi as c
    c.gemm_tuning_clear()
    yield c
    c.gemm_tuning_clear()


def _lines(path):
    with open(path) as f:
        return sorted(l.split() for l in f if l.strip() and not l.startswith("#"))


def test_tuning_table_round_trip(capi, tmp_path):
    src = tmp_path / "in.txt"
    src.write_text(GOOD)
    assert capi.gemm_tuning_load(str(src)) == capi.GEMM_OK
    assert capi.gemm_tuning_size() == 3
    out = tmp_path / "out.txt"
    assert capi.gemm_tuning_save(str(out)) == capi.GEMM_OK
    assert _lines(out) == _lines(src)
    # loading the same file again replaces, it does not duplicate
    assert capi.gemm_tuning_load(str(out)) == capi.GEMM_OK
    assert capi.gemm_tuning_size() == 3
    assert capi.gemm_tuning_clear() == capi.GEMM_OK
    assert capi.gemm_tuning_size() == 0


BAD_LINES = [
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 9 1 1 8 1.0",     # no plan 9
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 4 1 2 8 1.0",     # plan 4 takes no cluster split
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 1 2 2 8 1.0",     # two kinds of split at once
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 7 2 1 8 1.0",     # resident-A plan with a split
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 7 0 1 8 1.0",     # resident-A plan with stream-K
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 1 0 2 8 1.0",     # stream-K and a cluster split
    "gemmtune1 148 1 1024 1024 8192 0 0 0 3 1 1 1 1 1 1 1 8 1.0",     # unknown output type
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 1 1 3 8 1.0",     # cluster split of 3
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 1 1 1 8",         # missing time
    "gemmtune1 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 1 1 1 8 1.0 7",   # trailing field
    "gemmtune2 148 1 1024 1024 8192 0 0 0 1 1 1 1 1 1 1 1 8 1.0",     # unknown format
]


@pytest.mark.parametrize("bad", BAD_LINES)
def test_tuning_load_rejects_bad_files_whole(capi, tmp_path, bad):
    f = tmp_path / "bad.txt"
    f.write_text(GOOD + bad + "\n")
    assert capi.gemm_tuning_load(str(f)) == capi.GEMM_ERR_INVALID_ARG
    assert capi.gemm_tuning_size() == 0  # nothing from the file was loaded
    assert capi.gemm_tuning_load(str(tmp_path / "missing.txt")) == capi.GEMM_ERR_INVALID_ARG


def test_autotune_argument_checks_without_a_device(capi):
    assert capi.gemm_last_config() == (-1, 0, 0, 0)
    # unknown operand type or form, plain form with a batch, dedup without an index
    assert capi.gemm_autotune(2, 0, 1, 0, 4, 4, 4, 16, 4, 16, 4, 0, None, 16, 4, 0, 1, 1.0, 0.0, None)[0] == \
        capi.GEMM_ERR_INVALID_ARG
    assert capi.gemm_autotune(0, 3, 1, 0, 4, 4, 4, 16, 4, 16, 4, 0, None, 16, 4, 0, 1, 1.0, 0.0, None)[0] == \
        capi.GEMM_ERR_INVALID_ARG
    assert capi.gemm_autotune(0, 0, 2, 0, 4, 4, 4, 16, 4, 16, 4, 0, None, 16, 4, 0, 1, 1.0, 0.0, None)[0] == \
        capi.GEMM_ERR_INVALID_ARG
    assert capi.gemm_autotune(0, 2, 4, 2, 4, 4, 4, 16, 4, 16, 4, 16, None, 16, 4, 16, 1, 1.0, 0.0, None)[0] == \
        capi.GEMM_ERR_INVALID_ARG
    # bad sizes are rejected like the GEMM's; an empty problem has nothing to tune
    assert capi.gemm_autotune(0, 0, 1, 0, 4, 4, 8, 16, 7, 16, 8, 0, None, 16, 4, 0, 1, 1.0, 0.0, None)[0] == \
        capi.GEMM_ERR_INVALID_ARG
    assert capi.gemm_autotune(0, 0, 1, 0, 0, 4, 4, None, 4, None, 4, 0, None, None, 4, 0, 1, 1.0, 0.0, None)[0] == \
        capi.GEMM_OK
    assert capi.gemm_tuning_size() == 0


# ----------------------------------------------------------------------------- on a B200
def _table(capi, tmp_path):
    p = tmp_path / "t.txt"
    assert capi.gemm_tuning_save(str(p)) == capi.GEMM_OK
    return [l.split() for l in p.read_text().splitlines() if l.strip()]


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(1024, 1024, 8192), (2048, 2048, 2048), (300, 520, 3000)])
def test_autotune_then_calls_take_the_tuned_configuration(capi, tmp_path, shape):
    import torch

    import oracle
    from parity import check, to_dev_bf16, values_f64
    from synth import matrix_bf16
    M, N, K = shape
    A, B, c0 = matrix_bf16(191, M, K), matrix_bf16(192, N, K), matrix_bf16(193, M, N)
    dA, dB = to_dev_bf16(A), to_dev_bf16(B)
    C = to_dev_bf16(c0)
    C_before = C.clone()
    s = torch.cuda.current_stream().cuda_stream
    st, us = capi.gemm_autotune(0, 0, 1, 0, M, N, K, dA.data_ptr(), K, dB.data_ptr(), K, 0, None, C.data_ptr(), N, 0,
                                capi.GEMM_OUT_BF16, 0.5, 1.0, s)
    assert st == capi.GEMM_OK and us > 0
    assert torch.equal(C, C_before)  # the tuner writes only its scratch copy
    rows = _table(capi, tmp_path)
    assert len(rows) == 1
    row = rows[0]
    assert [int(x) for x in row[2:6]] == [1, M, N, K]
    tuned = tuple(int(x) for x in row[14:18])
    assert capi.gemm_bf16(M, N, K, dA.data_ptr(), K, dB.data_ptr(), K, C.data_ptr(), N, capi.GEMM_OUT_BF16,
                          0.5, 1.0, s) == capi.GEMM_OK
    torch.cuda.synchronize()
    assert capi.gemm_bf16_device_status(s) == capi.GEMM_OK
    assert capi.gemm_last_config() == tuned
    Cref, R = oracle.gemm(A, B, M=M, N=N, K=K, c0=c0, alpha=0.5, beta=1.0)
    assert check(values_f64(C), Cref, R, out_bf16=True)["ok"]


@pytest.mark.gpu
def test_autotune_batched_and_dedup_forms(capi, tmp_path):
    import torch

    from parity import to_dev_bf16
    from synth import matrix_bf16
    batch, M, N, K, n_u = 256, 256, 128, 512, 8
    W, X = to_dev_bf16(matrix_bf16(201, M, K)), to_dev_bf16(matrix_bf16(202, batch * K, N))
    Y = torch.empty((batch, M, N), dtype=torch.bfloat16, device="cuda")
    idx = torch.from_numpy((np.arange(batch) * n_u // batch).astype(np.int32)).cuda()
    s = torch.cuda.current_stream().cuda_stream
    st, _ = capi.gemm_autotune(0, 1, batch, 0, M, N, K, W.data_ptr(), K, X.data_ptr(), N, K * N, None, Y.data_ptr(),
                               N, M * N, capi.GEMM_OUT_BF16, 1.0, 0.0, s)
    assert st == capi.GEMM_OK
    st, _ = capi.gemm_autotune(0, 2, batch, n_u, M, N, K, W.data_ptr(), K, X.data_ptr(), N, K * N, idx.data_ptr(),
                               Y.data_ptr(), N, M * N, capi.GEMM_OUT_BF16, 1.0, 0.0, s)
    assert st == capi.GEMM_OK
    rows = _table(capi, tmp_path)
    assert sorted(int(r[6]) for r in rows) == [0, n_u]  # the two forms are separate problems
    dd = [r for r in rows if int(r[6]) == n_u][0]
    assert int(dd[15]) == 1 and int(dd[16]) == 1  # the deduplicated form never splits K
