"""Shared helpers of the GPU parity tests: seeded inputs on the device, the oracle on sampled
rows, and the element-wise tolerance checks.

Tolerances (float64 oracle values Cref, magnitude bound R = |alpha| sum|a||b| + |beta||c0|):
  fp32 output:  |C - Cref| <= 1e-3 * R + 1e-5                     (the stated fp32 bound)
  bf16 output:  |C - Cref| <= 8e-3 * |Cref| + 1e-3 * R + 1e-5      (per element),
                ||C - Cref||_F <= 8e-3 * ||Cref||_F                (normwise) and
                |C - Cref| <= 8e-3 * |Cref| wherever |Cref| >= 1e-2 * R
  fp16 output:  the first two with 1e-3 in place of 8e-3, the third with 2e-3 (fp16 rounding
                contributes at most 2^-11 |C| ~ 4.9e-4 |C|, fp32 accumulation up to ~1e-3 |C|
                at the floor |Cref| = 1e-2 R; no bound is stated for fp16, this one is derived)
The stated "relative error <= 8e-3" for bf16 output is ill-posed where Cref ~ 0 (cancellation),
so the per-element form adds the fp32 accumulation allowance; the normwise form and the check
over elements well above cancellation keep the 8e-3 relative bound as stated.  bf16 rounding
alone contributes at most 2^-9 |C| ~ 1.95e-3 |C|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from synth import bf16_bits_to_f64, matrix_bf16


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_f16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).cuda()


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def values_f64(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16))
    return t.to(torch.float64).numpy()


def sample_rows(M: int, seed: int = 0) -> list[int]:
    """Rows to check at full size.  In every 128-row block (the rows one CTA's accumulator
    holds): its first and last row, a random row, and one random row inside each 32-row lane
    quarter (each quarter is drained by a different epilogue warp); plus the matrix's last
    row.  Every output tile, both tile borders and all four epilogue warps are covered."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b0 in range(0, M, 128):
        b1 = min(M, b0 + 128)
        rows.update((b0, b1 - 1, int(rng.integers(b0, b1))))
        for q0 in range(b0, b1, 32):
            rows.add(int(rng.integers(q0, min(b1, q0 + 32))))
    rows.add(M - 1)
    return sorted(rows)


def check(C: np.ndarray, Cref: np.ndarray, R: np.ndarray, out_bf16: bool, out_f16: bool = False) -> dict:
    """Element-wise (and, for 16-bit outputs, normwise and relative-above-cancellation)
    tolerance check; returns a report."""
    err = np.abs(C - Cref)
    rel = 8e-3 if out_bf16 else 1e-3 if out_f16 else None
    if rel is not None:
        tol = rel * np.abs(Cref) + 1e-3 * R + 1e-5
    else:
        tol = 1e-3 * R + 1e-5
    bad = ~(err <= tol)  # NaN counts as bad
    nref = float(np.linalg.norm(Cref))
    rel_norm = float(np.linalg.norm(C - Cref) / nref) if nref > 0 else float(np.linalg.norm(C))
    big = np.abs(Cref) >= 1e-2 * R
    max_rel = float(np.nanmax(err[big] / np.abs(Cref[big]))) if big.any() else 0.0
    rep = {
        "n": int(C.size),
        "bad": int(bad.sum()),
        "max_err": float(np.nanmax(err)) if err.size else 0.0,
        "max_err_over_tol": float(np.nanmax(err / tol)) if err.size else 0.0,
        "rel_norm": rel_norm,
        "max_rel_above_cancellation": max_rel,
    }
    rel_floor = 8e-3 if out_bf16 else 2e-3
    rep["ok"] = rep["bad"] == 0 and (rel is None or (rel_norm <= rel and max_rel <= rel_floor))
    if rep["bad"]:
        idx = np.argwhere(bad)[:5]
        rep["first_bad"] = [(tuple(int(x) for x in i), float(C[tuple(i)]), float(Cref[tuple(i)]))
                            for i in idx]
    return rep


def make_inputs(M, N, K, *, seed_base, dist="normal", std_a=1.0, std_b=1.0, lda=None, ldb=None):
    A = matrix_bf16(seed_base + 0, M, K, dist=dist, std=std_a, ld=lda)
    B = matrix_bf16(seed_base + 1, N, K, dist=dist, std=std_b, ld=ldb)
    return A, B
