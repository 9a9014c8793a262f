"""Counter-based seeded generators for the synthetic GEMM inputs.

Definitions (all in numpy, vectorised, chunked to bound host memory):

* ``splitmix64(seed, i)`` -- the i-th output (i = 0, 1, ...) of Vigna's SplitMix64
  stream started at ``seed``: state_i = seed + (i+1)*0x9E3779B97F4A7C15 (mod 2^64),
  then the published two-multiply finaliser.  Counter-based, so any slice of a
  stream can be drawn without the prefix.
* ``uniform01_f64`` -- u = (x >> 11) * 2^-53, the top 53 bits of each output, in [0, 1).
* uniform on [-1, 1]  -- 2u - 1.
* ``normal_f64`` -- Box-Muller (the textbook polar-free form): element 2j and 2j+1 come
  from the pair (u_{2j}, u_{2j+1}) as r*cos(2*pi*u_{2j+1}) and r*sin(2*pi*u_{2j+1}) with
  r = sqrt(-2*ln(1 - u_{2j})), times the requested standard deviation.
* ``f64_to_bf16_bits`` -- round-to-nearest-even from the float64 value straight to
  bfloat16 (8 significant bits), returned as uint16 bit patterns.  No double rounding
  through float32.
* ``f64_to_f16_bits`` -- round-to-nearest-even from the float64 value straight to IEEE
  binary16 (11 significant bits for normal values; a fixed quantum of 2^-24 below 2^-14,
  the subnormal range), returned as uint16 bit patterns.

Seeds: base 20261202; matrix ``role`` r in {A:0, B:1, C:2} of workload ``index`` i uses
``seed = base + 16*i + r``.
"""
from __future__ import annotations

import numpy as np

BASE_SEED = 20261202
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

ROLES = {"A": 0, "B": 1, "C": 2, "W": 0, "X": 1, "Y": 2}


def seed_for(index: int, role: str) -> int:
    """Seed of matrix ``role`` ('A'/'B'/'C', or 'W'/'X'/'Y') of workload ``index``."""
    return BASE_SEED + 16 * int(index) + ROLES[role]


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs start..start+count-1 of the SplitMix64 stream seeded with ``seed``."""
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def uniform01_f64(seed: int, start: int, count: int) -> np.ndarray:
    """u in [0, 1) from the top 53 bits of each SplitMix64 output."""
    x = splitmix64(seed, start, count)
    return (x >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_f64(seed: int, start: int, count: int) -> np.ndarray:
    """Standard normals; element e of the stream uses draws 2*(e//2) and 2*(e//2)+1."""
    first_pair = start // 2
    last_pair = (start + count - 1) // 2
    npairs = last_pair - first_pair + 1
    u = uniform01_f64(seed, 2 * first_pair, 2 * npairs)
    u1 = u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u1))
    th = 2.0 * np.pi * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    off = start - 2 * first_pair
    return out[off:off + count]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even); uint16 bit patterns.

    Finite inputs only.  Values whose magnitude falls below the smallest normal bfloat16
    (2^-126) are not produced by these generators and are rejected.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite value")
    ax = np.abs(x)
    if np.any((ax != 0) & (ax < 2.0 ** -126)):
        raise ValueError("subnormal bf16 result not supported by the generator")
    bits = x.view(np.uint64)
    # float64 keeps 52 fraction bits, bfloat16 keeps 7: drop 45 with round-half-even.
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    with np.errstate(over="ignore"):
        rounded = (bits + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    y = rounded.view(np.float64)
    if np.any(np.abs(y) >= 2.0 ** 128):
        raise ValueError("value overflows bfloat16")
    f32 = y.astype(np.float32)  # exact: y has 8 significant bits and a float32 exponent
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def f64_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to IEEE binary16 (nearest, ties to even); uint16 bit patterns.

    Finite inputs whose rounded magnitude stays at most 65504 (the largest fp16) only.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite value")
    ax = np.abs(x)
    normal = ax >= 2.0 ** -14
    y = np.empty_like(x)
    # normal range: float64 keeps 52 fraction bits, fp16 keeps 10: drop 42, round half even
    bits = x[normal].view(np.uint64)
    lsb = (bits >> np.uint64(42)) & np.uint64(1)
    with np.errstate(over="ignore"):
        rounded = (bits + np.uint64((1 << 41) - 1) + lsb) & ~np.uint64((1 << 42) - 1)
    y[normal] = rounded.view(np.float64)
    # subnormal range: multiples of 2^-24; scaling by 2^24 is exact and rint rounds half even
    y[~normal] = np.rint(x[~normal] * 2.0 ** 24) * 2.0 ** -24
    if np.any(np.abs(y) > 65504.0):
        raise ValueError("value overflows fp16")
    # every y is now an fp16 value, so this conversion is exact
    return y.astype(np.float16).view(np.uint16)


def f16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    """Exact float64 value of fp16 bit patterns."""
    return np.ascontiguousarray(h, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    """Exact float64 value of bfloat16 bit patterns."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def matrix_bf16(seed: int, rows: int, cols: int, dist: str = "normal", std: float = 1.0,
                ld: int | None = None, dtype: str = "bf16") -> np.ndarray:
    """A rows x cols bfloat16 matrix (uint16 bits) drawn row-major from stream ``seed``.

    Element (r, c) is stream element r*cols + c, whatever ``ld``; with ``ld`` > cols the
    padding columns are filled with the bfloat16 NaN pattern 0x7FC1 so that a kernel that
    reads them shows up in the results.
    dist: 'normal' (mean 0, standard deviation ``std``) or 'uniform' (on [-1, 1]).
    dtype: 'bf16' (default) or 'f16' -- the 16-bit format the values are rounded to (the
    padding then holds the fp16 NaN pattern 0x7E01).
    """
    ld = cols if ld is None else ld
    if ld < cols:
        raise ValueError("ld < cols")
    if dtype not in ("bf16", "f16"):
        raise ValueError(dtype)
    to_bits = f64_to_bf16_bits if dtype == "bf16" else f64_to_f16_bits
    out = np.full((rows, ld), 0x7FC1 if dtype == "bf16" else 0x7E01, dtype=np.uint16)
    flat_total = rows * cols
    flat = np.empty(flat_total, dtype=np.uint16)
    for s in range(0, flat_total, _CHUNK):
        n = min(_CHUNK, flat_total - s)
        if dist == "normal":
            v = normal_f64(seed, s, n) * float(std)
        elif dist == "uniform":
            v = 2.0 * uniform01_f64(seed, s, n) - 1.0
        else:
            raise ValueError(dist)
        flat[s:s + n] = to_bits(v)
    out[:, :cols] = flat.reshape(rows, cols)
    return out


def matrix_f16(seed: int, rows: int, cols: int, dist: str = "normal", std: float = 1.0,
               ld: int | None = None) -> np.ndarray:
    """``matrix_bf16`` with the values rounded to fp16 instead (uint16 bit patterns)."""
    return matrix_bf16(seed, rows, cols, dist=dist, std=std, ld=ld, dtype="f16")
