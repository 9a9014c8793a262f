"""The fp64 oracle against its pins (CPU only), and proof that the pins bite."""
import pytest

import oracle
from oracle_pins import PINS, PLANTS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    ok, detail = pin()
    assert ok, detail


@pytest.mark.parametrize("plant", sorted(PLANTS), ids=[PLANTS[k] for k in sorted(PLANTS)])
def test_planted_mistake_fails_a_pin(plant, tmp_path):
    oracle.build(plant, str(tmp_path))
    failed = []
    for pin in PINS:
        ok, detail = pin(plant=plant, lib_dir=str(tmp_path))
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"planted mistake '{PLANTS[plant]}' passed every pin"


def test_oracle_rejects_bad_arguments():
    import numpy as np
    A = np.zeros((2, 2), np.uint16)
    with pytest.raises(ValueError):
        oracle.gemm(A, A, M=2, N=2, K=2, alpha=1.0, beta=1.0)  # beta != 0 without c0
