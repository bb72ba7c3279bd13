"""Plant plausible mistakes in the oracle (compile-time variants of its C
source, CPU only) and check that the pins catch every one of them.

Mutants (see the LO_MUTANT blocks in oracle/lapsum_oracle.c):
  1  the prefix recurrence drops its "+1" term
  2  the suffix recurrence uses the wrong sign in its exponent
  3  the closed-form root ignores the sign of mu (one anchor for all cases)
  4  the backward pass drops the budget term lambda
  5  dL/dalpha ignores that the threshold moves with alpha
  6  the bracket's rank half-width drops the (1 - q) factor of the binomial variance
  7  the bracket's half-width is applied below the mean only
"""
import os

import numpy as np
import pytest

import oracle as oracle_mod
from tests import test_oracle_pins as pins


def _battery(o):
    """Run a handful of pins against oracle `o`; return the failures."""
    fails = []

    def run(name, fn):
        try:
            fn()
        except (AssertionError, oracle_mod.OracleError, FloatingPointError, ValueError) as e:
            fails.append((name, repr(e)[:120]))

    for seed in range(12):
        run(f"brute{seed}", lambda s=seed: pins.test_brute_force_tiny(o, s))
    run("budget", lambda: pins.test_budget_sum(o))
    run("pair", lambda: pins.test_symmetric_pair(o, 3.0, 0.01))
    run("c1", lambda: pins.test_threshold_c1_bisection(o))
    run("bwd", lambda: pins.test_backward_invariants(o))
    for seed in range(2):
        run(f"fd{seed}", lambda s=seed: pins.test_vjp_finite_differences(o, s))
        run(f"fda{seed}", lambda s=seed: pins.test_alpha_gradient_finite_differences(o, s))
    run("apair", lambda: pins.test_alpha_gradient_symmetric_pair(o))
    run("aconst", lambda: pins.test_alpha_gradient_constant_upstream_is_zero(o))
    run("ranks", lambda: pins.check_rank_miss_probabilities(o))
    run("misses", lambda: pins.check_bracket_miss_rates(o, cases=pins.MISS_CASES[2:]))
    return fails


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6, 7])
def test_pins_catch_mutant(tmp_path, mutant):
    path = oracle_mod.build(out=str(tmp_path / f"liblo_m{mutant}.so"), mutant=mutant, force=True)
    o = oracle_mod.Oracle(oracle_mod.load(path))
    with np.errstate(all="ignore"):
        fails = _battery(o)
    assert fails, f"mutant {mutant} slipped through every pin"


def test_clean_oracle_passes_battery(orc):
    assert _battery(orc) == []
