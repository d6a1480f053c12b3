"""Pins of the fp64 oracle (CPU only).

Every pin family in ``oracle_pins`` must pass on the real oracle, and every
build with a planted mistake (``-DORACLE_MUTANT=n``) must fail at least one
of them, which shows the pins can tell a plausible slip from the definition.
"""
import numpy as np
import pytest

import oracle
from oracle import sdpa_oracle
from tests import oracle_pins as pins

MUTANTS = {
    1: "causal bound off by one",
    2: "window one key too wide",
    3: "strided GQA head mapping",
    4: "causal aligned to the start of the keys",
    5: "scale dropped",
    6: "V rows reversed",
    7: "missing normalisation",
}


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin_passes(pin):
    fails = pin(0)
    assert not fails, fails


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_planted_mistake_is_caught(mutant):
    lib = oracle.load_oracle(mutant)
    assert lib.oracle_mutant_id() == mutant
    caught = [p.__name__ for p in pins.ALL_PINS if p(mutant)]
    assert caught, f"no pin catches mutant {mutant} ({MUTANTS[mutant]})"


def test_row_subset_matches_full():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((2, 4, 20, 16))
    k = rng.standard_normal((2, 2, 30, 16))
    v = rng.standard_normal((2, 2, 30, 8))
    full = sdpa_oracle(q, k, v, 0.25, True, 6)
    rows = [0, 7, 19, 3]
    sub = sdpa_oracle(q, k, v, 0.25, True, 6, rows=rows)
    assert np.array_equal(sub, full[:, :, rows])


def test_threads_do_not_change_result():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 8, 33, 24))
    k = rng.standard_normal((1, 2, 70, 24))
    v = rng.standard_normal((1, 2, 70, 24))
    a = sdpa_oracle(q, k, v, 0.2, True, 0, nthreads=1)
    b = sdpa_oracle(q, k, v, 0.2, True, 0, nthreads=7)
    assert np.array_equal(a, b)


def test_invalid_arguments_rejected():
    q = np.zeros((1, 3, 4, 8))
    k = np.zeros((1, 2, 4, 8))
    with pytest.raises(ValueError):
        sdpa_oracle(q, k, k, 1.0)  # Hq not a multiple of Hkv
    q = np.zeros((1, 2, 4, 8))
    with pytest.raises(ValueError):
        sdpa_oracle(q, k, k, 1.0, key_range=(3, 9))
    with pytest.raises(ValueError):
        sdpa_oracle(q, k, k, 1.0, rows=[4])


def test_empty_key_range_gives_zero_weight():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 2, 3, 8))
    k = rng.standard_normal((1, 1, 10, 8))
    o, lse = sdpa_oracle(q, k, k, 0.3, True, 0, key_range=(9, 10), return_lse=True)
    # rows 0 and 1 sit at positions 7 and 8: key 9 is in their future
    assert np.all(o[:, :, :2] == 0) and np.all(np.isneginf(lse[:, :, :2]))
    assert np.all(np.isfinite(lse[:, :, 2]))
