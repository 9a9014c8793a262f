"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each ``pin_*`` returns ``(ok, detail)`` for the oracle build ``plant`` (0 = the real
oracle; 1..8 = copies with one planted mistake).  tests/test_oracle.py asserts that the
real oracle passes every pin and that every planted copy fails at least one.

What pins what:
  golden        hand-worked examples in tests/golden (alpha/beta, signs, both B layouts)
  identity      A = I gives C = B^T exactly; B = I gives C = A exactly
  permutation   a permutation matrix permutes the other operand's rows/columns exactly
  rank1         a(i,k)=u_i s_k, b(k,j)=v_j t_k gives u_i v_j (s.t) in closed form
  integer       small-integer inputs agree exactly with an int64 matrix product
  fraction      tiny random bf16 inputs agree with exact rational arithmetic within
                K * 2^-53 * R (the float64 summation bound)
  alpha_beta    alpha = 0 gives beta*c0; beta = 0 ignores a NaN c0
  symmetry      (A B^T)^T equals B A^T exactly
  layouts       an N-major B gives the same result as its K-major transpose
  rows          a row subset equals the same rows of the full result
  batched       the batched call equals the single GEMM on each batch slice, and
                exact rationals on a tiny batch
  f16_decode    every one of the 65536 fp16 bit patterns decodes to numpy's float16 value
  f16_golden    a hand-worked fp16 example (10-bit fractions, subnormal, 4096, c0 in fp16)
  f16_integer   integer fp16 inputs beyond bf16's exact range agree with an int64 product
  f16_fraction  tiny random fp16 inputs agree with exact rational arithmetic
  dedup         the deduplicated shared-W form (items share distinct entries by index) equals
                exact rationals per item on a tiny case, gives identical rows to items that
                share an entry, and equals the batched form on the explicitly expanded batch
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

import oracle
from synth import (bf16_bits_to_f64, f16_bits_to_f64, f64_to_bf16_bits, f64_to_f16_bits, matrix_bf16,
                   matrix_f16)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
U53 = 2.0 ** -53


def _bf(vals, shape):
    return f64_to_bf16_bits(np.asarray(vals, dtype=np.float64)).reshape(shape)


def _read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            d[key] = [float(v) for v in vals]
    return d


def pin_golden(plant=0, lib_dir=None):
    d = _read_golden("gemm_hand_2x2x3.txt")
    M, N, K = int(d["M"][0]), int(d["N"][0]), int(d["K"][0])
    A = _bf(d["A"], (M, K))
    Bs = _bf(d["Bs"], (N, K))
    C0 = np.asarray(d["C0"], dtype=np.float32).reshape(M, N)
    C, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, c0=C0, alpha=d["alpha"][0], beta=d["beta"][0],
                       plant=plant, lib_dir=lib_dir)
    ok1 = np.array_equal(C, np.asarray(d["C"]).reshape(M, N))
    d = _read_golden("gemm_hand_signed_3x1x2.txt")
    M, N, K = int(d["M"][0]), int(d["N"][0]), int(d["K"][0])
    A = _bf(d["A"], (M, K))
    Bn = _bf(d["Bn"], (K, N))
    C0 = _bf(d["C0"], (M, N))
    C, _ = oracle.gemm(A, Bn, M=M, N=N, K=K, b_kmajor=False, c0=C0, alpha=d["alpha"][0],
                       beta=d["beta"][0], plant=plant, lib_dir=lib_dir)
    ok2 = np.array_equal(C, np.asarray(d["C"]).reshape(M, N))
    return ok1 and ok2, f"hand examples: {ok1}, {ok2}"


def pin_identity(plant=0, lib_dir=None):
    n, m = 24, 13
    eye = _bf(np.eye(n), (n, n))
    Bs = matrix_bf16(11, m, n)  # N=m x K=n
    C, _ = oracle.gemm(eye, Bs, M=n, N=m, K=n, plant=plant, lib_dir=lib_dir)
    ok1 = np.array_equal(C, bf16_bits_to_f64(Bs).T)
    A = matrix_bf16(12, m, n)  # M=m x K=n
    C, _ = oracle.gemm(A, eye, M=m, N=n, K=n, plant=plant, lib_dir=lib_dir)
    ok2 = np.array_equal(C, bf16_bits_to_f64(A))
    return ok1 and ok2, f"A=I: {ok1}, B=I: {ok2}"


def pin_permutation(plant=0, lib_dir=None):
    rng = np.random.default_rng(5)
    n, m = 17, 9
    p = rng.permutation(n)
    P = np.zeros((n, n))
    P[np.arange(n), p] = 1.0  # (P X)[i] = X[p[i]]
    Pb = _bf(P, (n, n))
    Bs = matrix_bf16(13, m, n)  # b(k,j) = Bs[j][k]
    C, _ = oracle.gemm(Pb, Bs, M=n, N=m, K=n, plant=plant, lib_dir=lib_dir)
    ok1 = np.array_equal(C, bf16_bits_to_f64(Bs).T[p, :])
    A = matrix_bf16(14, m, n)
    C, _ = oracle.gemm(A, Pb, M=m, N=n, K=n, plant=plant, lib_dir=lib_dir)
    # b(k,j) = P[j][k] = [k == p[j]]  ->  C[i][j] = a(i, p[j])
    ok2 = np.array_equal(C, bf16_bits_to_f64(A)[:, p])
    return ok1 and ok2, f"row perm: {ok1}, col perm: {ok2}"


def pin_rank1(plant=0, lib_dir=None):
    rng = np.random.default_rng(7)
    M, N, K = 11, 10, 37
    u = rng.integers(-3, 4, M).astype(float)
    s = rng.integers(-3, 4, K).astype(float)
    v = rng.integers(-3, 4, N).astype(float)
    t = rng.integers(-3, 4, K).astype(float)
    A = _bf(np.outer(u, s), (M, K))
    Bs = _bf(np.outer(v, t), (N, K))
    c0 = rng.integers(-4, 5, (M, N)).astype(np.float32)
    alpha, beta = 0.25, 3.0
    C, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, c0=c0, alpha=alpha, beta=beta, plant=plant,
                       lib_dir=lib_dir)
    closed = alpha * np.outer(u, v) * float(np.dot(s, t)) + beta * c0.astype(float)
    return np.array_equal(C, closed), "rank-1 closed form"


def pin_integer(plant=0, lib_dir=None):
    rng = np.random.default_rng(9)
    M, N, K = 33, 29, 2048
    Ai = rng.integers(-2, 3, (M, K))
    Bi = rng.integers(-2, 3, (N, K))
    A = _bf(Ai, (M, K))
    Bs = _bf(Bi, (N, K))
    C, R = oracle.gemm(A, Bs, M=M, N=N, K=K, plant=plant, lib_dir=lib_dir)
    exact = Ai.astype(np.int64) @ Bi.astype(np.int64).T
    rexact = np.abs(Ai).astype(np.int64) @ np.abs(Bi).astype(np.int64).T
    return np.array_equal(C, exact) and np.array_equal(R, rexact), "integer inputs"


def _exact_gemm(a, b_kn, c0, alpha, beta):
    """Exact rationals: a (M x K), b_kn (K x N) float arrays of exact bf16 values."""
    M, K = a.shape
    N = b_kn.shape[1]
    out = [[None] * N for _ in range(M)]
    bound = [[None] * N for _ in range(M)]
    fa, fb = Fraction(alpha), Fraction(beta)
    for i in range(M):
        for j in range(N):
            s = Fraction(0)
            r = Fraction(0)
            for k in range(K):
                p = Fraction(a[i, k]) * Fraction(b_kn[k, j])
                s += p
                r += abs(p)
            c = Fraction(float(c0[i, j])) if (c0 is not None and beta != 0) else Fraction(0)
            out[i][j] = fa * s + fb * c
            bound[i][j] = abs(fa) * r + abs(fb) * abs(c)
    return out, bound


def pin_fraction(plant=0, lib_dir=None):
    rng = np.random.default_rng(11)
    worst = 0.0
    for trial in range(24):
        M, N, K = (int(x) for x in rng.integers(1, 10, 3))
        if trial < 3:
            K = 1
        kmajor = bool(trial % 2)
        A = matrix_bf16(100 + trial, M, K)
        if kmajor:
            B = matrix_bf16(200 + trial, N, K)
            b_kn = bf16_bits_to_f64(B).T
        else:
            B = matrix_bf16(200 + trial, K, N)
            b_kn = bf16_bits_to_f64(B)
        alpha = float(rng.choice([1.0, 0.5, -1.5, 3.0]))
        beta = float(rng.choice([0.0, 1.0, -0.75]))
        if trial % 3 == 0:
            c0 = matrix_bf16(300 + trial, M, N)
            c0v = bf16_bits_to_f64(c0)
        else:
            c0 = (rng.standard_normal((M, N))).astype(np.float32)
            c0v = c0.astype(np.float64)
        C, R = oracle.gemm(A, B, M=M, N=N, K=K, b_kmajor=kmajor, c0=c0, alpha=alpha,
                           beta=beta, plant=plant, lib_dir=lib_dir)
        ex, bd = _exact_gemm(bf16_bits_to_f64(A), b_kn, c0v, alpha, beta)
        for i in range(M):
            for j in range(N):
                err = abs(Fraction(C[i, j]) - ex[i][j])
                tol = Fraction(K + 2) * Fraction(U53) * bd[i][j]
                if err > tol:
                    return False, f"trial {trial} ({M},{N},{K}) elem ({i},{j}) err {float(err)}"
                if abs(Fraction(R[i, j]) - bd[i][j]) > tol:
                    return False, f"trial {trial}: bound R wrong at ({i},{j})"
                if bd[i][j] > 0:
                    worst = max(worst, float(err / bd[i][j]))
    return True, f"worst err/R = {worst:.3g}"


def pin_alpha_beta(plant=0, lib_dir=None):
    M, N, K = 7, 6, 19
    A = matrix_bf16(21, M, K)
    Bs = matrix_bf16(22, N, K)
    c0 = matrix_bf16(23, M, N)
    C, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, c0=c0, alpha=0.0, beta=-1.5, plant=plant,
                       lib_dir=lib_dir)
    ok1 = np.array_equal(C, -1.5 * bf16_bits_to_f64(c0))
    nanc = np.full((M, N), np.nan, dtype=np.float32)
    C2, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, c0=nanc, alpha=1.0, beta=0.0, plant=plant,
                        lib_dir=lib_dir)
    C3, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, plant=plant, lib_dir=lib_dir)
    ok2 = bool(np.all(np.isfinite(C2))) and np.array_equal(C2, C3)
    return ok1 and ok2, f"alpha=0: {ok1}, beta=0 ignores NaN: {ok2}"


def pin_symmetry(plant=0, lib_dir=None):
    M, N, K = 21, 14, 45
    A = matrix_bf16(31, M, K)
    Bs = matrix_bf16(32, N, K)
    C1, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, plant=plant, lib_dir=lib_dir)
    C2, _ = oracle.gemm(Bs, A, M=N, N=M, K=K, plant=plant, lib_dir=lib_dir)
    return np.array_equal(C1, C2.T), "(A B^T)^T == B A^T"


def pin_layouts(plant=0, lib_dir=None):
    M, N, K = 12, 20, 33
    A = matrix_bf16(41, M, K)
    Bs = matrix_bf16(42, N, K)
    Bn = np.ascontiguousarray(Bs.T)
    C1, R1 = oracle.gemm(A, Bs, M=M, N=N, K=K, b_kmajor=True, plant=plant, lib_dir=lib_dir)
    C2, R2 = oracle.gemm(A, Bn, M=M, N=N, K=K, b_kmajor=False, plant=plant, lib_dir=lib_dir)
    # padded leading dimensions must not change anything
    Ap = matrix_bf16(41, M, K, ld=K + 7)
    C3, _ = oracle.gemm(Ap, Bs, M=M, N=N, K=K, plant=plant, lib_dir=lib_dir)
    ok = np.array_equal(C1, C2) and np.array_equal(R1, R2) and np.array_equal(C1, C3)
    return ok, "K-major == N-major; padded lda"


def pin_rows(plant=0, lib_dir=None):
    M, N, K = 40, 9, 31
    A = matrix_bf16(51, M, K)
    Bs = matrix_bf16(52, N, K)
    rows = [39, 0, 17, 17, 5]
    C, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, plant=plant, lib_dir=lib_dir)
    Cs, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, rows=rows, plant=plant, lib_dir=lib_dir)
    return np.array_equal(Cs, C[rows]), "row subset"


def pin_batched(plant=0, lib_dir=None):
    batch, M, N, K = 3, 5, 4, 6
    W = matrix_bf16(61, M, K)
    X = matrix_bf16(62, batch * K, N)  # X[b] = rows b*K .. b*K+K-1
    y0 = matrix_bf16(63, batch * M, N)
    Cb, _ = oracle.gemm_batched(W, X, batch=batch, M=M, N=N, K=K, stride_x=K * N, y0=y0,
                                stride_y=M * N, alpha=0.5, beta=2.0, plant=plant,
                                lib_dir=lib_dir)
    ok = True
    for b in range(batch):
        xb = X[b * K:(b + 1) * K]
        Cs, _ = oracle.gemm(W, xb, M=M, N=N, K=K, b_kmajor=False,
                            c0=y0[b * M:(b + 1) * M], alpha=0.5, beta=2.0, plant=plant,
                            lib_dir=lib_dir)
        ok = ok and np.array_equal(Cb[b], Cs)
        ex, bd = _exact_gemm(bf16_bits_to_f64(W), bf16_bits_to_f64(xb),
                             bf16_bits_to_f64(y0[b * M:(b + 1) * M]), 0.5, 2.0)
        for i in range(M):
            for j in range(N):
                if abs(Fraction(Cb[b, i, j]) - ex[i][j]) > (K + 2) * Fraction(U53) * bd[i][j]:
                    ok = False
    return ok, "batched == per-slice and exact"


def pin_f16_decode(plant=0, lib_dir=None):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(h, "f16", plant=plant, lib_dir=lib_dir)
    want = h.view(np.float16).astype(np.float64)  # numpy's own binary16 conversion
    nan = np.isnan(want)
    ok = np.array_equal(np.isnan(got), nan) and np.array_equal(got[~nan], want[~nan])
    # signed zeros keep their sign
    ok = ok and np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))
    return ok, "all fp16 patterns"


def _f16(vals, shape):
    return f64_to_f16_bits(np.asarray(vals, dtype=np.float64)).reshape(shape)


def pin_f16_golden(plant=0, lib_dir=None):
    d = _read_golden("gemm_hand_f16_1x2x3.txt")
    M, N, K = int(d["M"][0]), int(d["N"][0]), int(d["K"][0])
    A = _f16(d["A"], (M, K))
    Bs = _f16(d["Bs"], (N, K))
    # the fixture's values must be fp16 values as written (no rounding on the way in)
    ok0 = (np.array_equal(f16_bits_to_f64(A).ravel(), d["A"])
           and np.array_equal(f16_bits_to_f64(Bs).ravel(), d["Bs"]))
    C0 = np.asarray(d["C0"], dtype=np.float16).reshape(M, N)
    C, _ = oracle.gemm(A, Bs, M=M, N=N, K=K, c0=C0, alpha=d["alpha"][0], beta=d["beta"][0],
                       plant=plant, lib_dir=lib_dir, in_dtype="f16")
    ok = ok0 and np.array_equal(C, np.asarray(d["C"]).reshape(M, N))
    return ok, f"fp16 hand example: {ok}"


def pin_f16_integer(plant=0, lib_dir=None):
    rng = np.random.default_rng(19)
    M, N, K = 21, 18, 1024
    Ai = rng.integers(-300, 301, (M, K))  # exact in fp16 (11 significant bits), not in bf16
    Bi = rng.integers(-300, 301, (N, K))
    A = _f16(Ai, (M, K))
    Bs = _f16(Bi, (N, K))
    C, R = oracle.gemm(A, Bs, M=M, N=N, K=K, plant=plant, lib_dir=lib_dir, in_dtype="f16")
    exact = Ai.astype(np.int64) @ Bi.astype(np.int64).T
    rexact = np.abs(Ai).astype(np.int64) @ np.abs(Bi).astype(np.int64).T
    return np.array_equal(C, exact) and np.array_equal(R, rexact), "integer fp16 inputs"


def pin_f16_fraction(plant=0, lib_dir=None):
    rng = np.random.default_rng(23)
    for trial in range(12):
        M, N, K = (int(x) for x in rng.integers(1, 8, 3))
        kmajor = bool(trial % 2)
        A = matrix_f16(400 + trial, M, K, std=0.01 if trial % 3 == 0 else 1.0)  # subnormals too
        B = matrix_f16(500 + trial, N, K) if kmajor else matrix_f16(500 + trial, K, N)
        b_kn = f16_bits_to_f64(B).T if kmajor else f16_bits_to_f64(B)
        alpha = float(rng.choice([1.0, -0.5, 2.0]))
        beta = float(rng.choice([0.0, 1.0, -0.25]))
        c0 = matrix_f16(600 + trial, M, N).view(np.float16)
        C, R = oracle.gemm(A, B, M=M, N=N, K=K, b_kmajor=kmajor, c0=c0, alpha=alpha, beta=beta,
                           plant=plant, lib_dir=lib_dir, in_dtype="f16")
        ex, bd = _exact_gemm(f16_bits_to_f64(A), b_kn, c0.astype(np.float64), alpha, beta)
        for i in range(M):
            for j in range(N):
                tol = Fraction(K + 2) * Fraction(U53) * bd[i][j]
                if abs(Fraction(C[i, j]) - ex[i][j]) > tol or abs(Fraction(R[i, j]) - bd[i][j]) > tol:
                    return False, f"trial {trial} ({M},{N},{K}) elem ({i},{j})"
    return True, "fp16 exact rationals"


def pin_dedup(plant=0, lib_dir=None):
    n_x, M, N, K = 3, 4, 5, 7
    index = [2, 0, 2, 1, 2, 0]  # six items over three distinct entries
    W = matrix_bf16(71, M, K)
    X = matrix_bf16(72, n_x * K, N)
    y0 = matrix_bf16(73, len(index) * M, N)
    C, _ = oracle.gemm_batched_dedup(W, X, index, n_x=n_x, M=M, N=N, K=K, stride_x=K * N, y0=y0,
                                     stride_y=M * N, alpha=-0.5, beta=1.0, plant=plant, lib_dir=lib_dir)
    ok = True
    for b, u in enumerate(index):
        ex, bd = _exact_gemm(bf16_bits_to_f64(W), bf16_bits_to_f64(X[u * K:(u + 1) * K]),
                             bf16_bits_to_f64(y0[b * M:(b + 1) * M]), -0.5, 1.0)
        for i in range(M):
            for j in range(N):
                if abs(Fraction(C[b, i, j]) - ex[i][j]) > (K + 2) * Fraction(U53) * bd[i][j]:
                    ok = False
    # items 0, 2 and 4 share entry 2: with beta = 0 their rows are identical
    C0, _ = oracle.gemm_batched_dedup(W, X, index, n_x=n_x, M=M, N=N, K=K, stride_x=K * N,
                                      plant=plant, lib_dir=lib_dir)
    same = np.array_equal(C0[0], C0[2]) and np.array_equal(C0[0], C0[4]) and np.array_equal(C0[1], C0[5])
    # the batched form on the expanded batch X[b] = X[index[b]]
    Xe = np.concatenate([X[u * K:(u + 1) * K] for u in index])
    Ce, _ = oracle.gemm_batched(W, Xe, batch=len(index), M=M, N=N, K=K, stride_x=K * N, plant=plant,
                                lib_dir=lib_dir)
    return ok and same and np.array_equal(C0, Ce), f"exact: {ok}, shared rows: {same}"


PINS = [pin_golden, pin_identity, pin_permutation, pin_rank1, pin_integer, pin_fraction,
        pin_alpha_beta, pin_symmetry, pin_layouts, pin_rows, pin_batched, pin_f16_decode,
        pin_f16_golden, pin_f16_integer, pin_f16_fraction, pin_dedup]
PLANTS = {
    1: "last k term dropped",
    2: "wrong sign on the beta term",
    3: "operand B read transposed",
    4: "alpha also scales the old C",
    5: "output row taken from the next row of A",
    6: "column index off by one",
    7: "running sums rounded to float32",
    8: "first k term dropped",
    9: "fp16 exponent bias off by one",
    10: "dedup: item position used instead of its distinct entry",
}
