"""The seeded input generators against their published definitions (CPU only)."""
import math
from fractions import Fraction

import numpy as np

from synth import (bf16_bits_to_f64, f16_bits_to_f64, f64_to_bf16_bits, f64_to_f16_bits, matrix_bf16,
                   matrix_f16, normal_f64, seed_for, splitmix64, uniform01_f64)


def test_splitmix64_published_vectors():
    # SplitMix64 seeded with 0: the first three outputs of the reference implementation.
    out = splitmix64(0, 0, 3)
    assert [int(x) for x in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                     0x06C45D188009454F]


def test_splitmix64_is_counter_based():
    full = splitmix64(12345, 0, 1000)
    assert np.array_equal(full[300:700], splitmix64(12345, 300, 400))


def test_uniform_and_normal_slices_agree():
    assert np.array_equal(uniform01_f64(7, 0, 101)[33:77], uniform01_f64(7, 33, 44))
    assert np.array_equal(normal_f64(7, 0, 101)[33:78], normal_f64(7, 33, 45))


def _bf16_rne_exact(x: float) -> float:
    """Nearest bfloat16 by exhaustive neighbour search on exact rationals, ties to even."""
    if x == 0:
        return 0.0
    m, e = math.frexp(abs(x))  # |x| = m * 2^e, m in [0.5, 1)
    ulp = Fraction(2) ** (e - 8)  # 8 significant bits
    q = Fraction(abs(x)) / ulp
    lo = math.floor(q)
    frac = q - lo
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return math.copysign(float(lo * ulp), x)


def test_bf16_rounding_matches_exact_rne():
    rng = np.random.default_rng(3)
    vals = list(rng.standard_normal(2000) * 10.0 ** rng.integers(-5, 5, 2000))
    # exact ties and near-ties around 1.0 (bf16 ulp at 1 is 2^-7)
    t = 2.0 ** -8
    vals += [1 + t, 1 + 3 * t, 1 - t / 2, -(1 + t), 1 + t + 2.0 ** -40, 1 + t - 2.0 ** -40,
             3.0, -0.0, 0.0, 65504.0, 1e30]
    got = bf16_bits_to_f64(f64_to_bf16_bits(np.array(vals)))
    want = np.array([_bf16_rne_exact(v) for v in vals])
    assert np.array_equal(got, want)


def test_matrix_statistics_and_padding():
    a = bf16_bits_to_f64(matrix_bf16(seed_for(2, "A"), 512, 512))
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    w = bf16_bits_to_f64(matrix_bf16(seed_for(3, "B"), 256, 512, std=0.02))
    assert abs(w.std() - 0.02) < 0.0005
    u = bf16_bits_to_f64(matrix_bf16(seed_for(0, "A"), 256, 256, dist="uniform"))
    assert u.min() >= -1.0 and u.max() <= 1.0 and abs(u.mean()) < 0.01
    p = matrix_bf16(5, 3, 5, ld=8)
    assert np.array_equal(p[:, :5], matrix_bf16(5, 3, 5)) and np.all(p[:, 5:] == 0x7FC1)


def test_seeds_are_distinct_per_role_and_workload():
    seeds = {seed_for(i, r) for i in range(5) for r in "ABC"}
    assert len(seeds) == 15


def _f16_rne_exact(x: float) -> float:
    """Nearest fp16 on exact rationals, ties to even: 11 significant bits for normal values,
    a fixed quantum of 2^-24 below the smallest normal 2^-14."""
    if x == 0:
        return 0.0
    m, e = math.frexp(abs(x))  # |x| = m * 2^e, m in [0.5, 1)
    ulp = Fraction(2) ** (e - 11) if abs(x) >= 2.0 ** -14 else Fraction(2) ** -24
    q = Fraction(abs(x)) / ulp
    lo = math.floor(q)
    frac = q - lo
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return math.copysign(float(lo * ulp), x)


def test_f16_rounding_matches_exact_rne_and_numpy():
    rng = np.random.default_rng(4)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-7, 4, 3000))
    t = 2.0 ** -11  # half an fp16 ulp at 1
    s = 2.0 ** -25  # half the subnormal quantum
    vals += [1 + t, 1 + 3 * t, -(1 + t), 1 + t + 2.0 ** -40, 1 + t - 2.0 ** -40, s, 3 * s, -5 * s,
             2.0 ** -14 - s, 2.0 ** -14 + s, 65504.0, 65519.0, -0.0, 0.0, 0.1, 2.0 ** -24]
    got = f16_bits_to_f64(f64_to_f16_bits(np.array(vals)))
    want = np.array([_f16_rne_exact(v) for v in vals])
    assert np.array_equal(got, want)
    # numpy rounds float64 to float16 directly, also to nearest even
    assert np.array_equal(got, np.array(vals).astype(np.float16).astype(np.float64))


def test_f16_matrix_padding_and_statistics():
    w = f16_bits_to_f64(matrix_f16(seed_for(2, "B"), 256, 512, std=0.02))
    assert abs(w.std() - 0.02) < 0.0005
    p = matrix_f16(5, 3, 5, ld=8)
    assert np.array_equal(p[:, :5], matrix_f16(5, 3, 5)) and np.all(p[:, 5:] == 0x7E01)
    assert np.isnan(p[:, 5:].view(np.float16)).all()
