"""Planted mistakes in the oracle must be caught by its pins.

The oracle carries a test-only switch that plants one plausible mistake at a
time (dropped 1/sqrt(d) scale, interleaved query->KV head map, sum instead of
mean over heads, reversed tie rule).  Each must make at least one pin of
test_oracle_pins fail; the switch is reset afterwards.
"""
import pytest

import test_oracle_pins as pins

CHECKS = [
    lambda o: pins.test_dense_equals_torch_sdpa(o, 65, 8, 2, 32),
    lambda o: pins.test_mass_rows_sum_to_one(o, 70, 8, 2, 32),
    lambda o: pins.test_zero_queries_closed_form(o),
    lambda o: pins.test_brute_force_tiny(o, 24, 4, 2, 8, 3),
]


@pytest.mark.parametrize("mutation", [1, 2, 3, 4])
def test_planted_mistake_is_caught(oracle_mod, mutation):
    caught = 0
    oracle_mod.set_mutation(mutation)
    try:
        for chk in CHECKS:
            try:
                chk(oracle_mod)
            except AssertionError:
                caught += 1
    finally:
        oracle_mod.set_mutation(0)
    assert caught >= 1, f"planted mistake {mutation} passed every pin"


def test_clean_oracle_passes_the_same_checks(oracle_mod):
    oracle_mod.set_mutation(0)
    for chk in CHECKS:
        chk(oracle_mod)
