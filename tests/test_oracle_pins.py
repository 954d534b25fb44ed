"""The CPU oracle against hand-worked examples, closed forms and invariants."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import oracle_pins
from helpers import load_golden, random_problem


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin()


def test_golden_matches_exact_rational_bruteforce():
    """The hand-worked numbers of the L2-off golden agree exactly with an
    exact-rational brute force of the same two tokens."""
    name = "k4v4_two_tokens_decay_quarter.json"
    case = load_golden(name)
    outs, states = oracle_pins.golden_exact_rational(name)
    assert outs == [[Fraction(x) for x in row] for row in case["expected_out"]]
    assert states == [[[Fraction(x) for x in row] for row in st] for st in case["expected_inter"]]


def test_fp32_drift_is_far_below_state_tolerance(oracle_lib):
    """Sizing: a correct fp32 evaluation of 64 chained tokens at K = V = 128
    stays within ~1e-6 of fp64 on the state, well inside the 1e-4 bar, and
    the outputs within the bf16 output bar."""
    rng = np.random.default_rng(30)
    p = random_problem(rng, lens=[64, 33], H=1, HV=2, K=128, V=128)
    _, o64, s64, _ = oracle.update(*(p[k] for k in ("q", "k", "v", "a", "b", "A_log", "dt_bias",
                                                      "state_pool", "state_indices", "cu_seqlens")))
    _, o32, s32, _ = oracle.update(*(p[k] for k in ("q", "k", "v", "a", "b", "A_log", "dt_bias",
                                                      "state_pool", "state_indices", "cu_seqlens")),
                                   precision="f32")
    assert np.max(np.abs(s32 - s64)) < 1e-5
    assert np.all(np.abs(o32 - o64) <= 1e-3 * (1 + np.abs(o64)))


def test_oracle_rejects_bad_arguments(oracle_lib):
    rng = np.random.default_rng(31)
    p = random_problem(rng, lens=[1], H=2, HV=3, K=8, V=8)   # HV % H != 0
    with pytest.raises(ValueError):
        oracle.update(*(p[k] for k in ("q", "k", "v", "a", "b", "A_log", "dt_bias",
                                       "state_pool", "state_indices", "cu_seqlens")))
