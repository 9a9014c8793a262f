"""The seeded input generators against their published definitions (CPU only)."""
import math
from fractions import Fraction

import numpy as np

from synth import (bf16_bits_to_f64, f64_to_bf16_bits, matrix_bf16, normal_f64, seed_for,
                   splitmix64, uniform01_f64)


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
