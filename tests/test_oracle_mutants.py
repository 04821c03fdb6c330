"""Mutation self-test: the oracle pins must reject plausible mistakes.

Each ORACLE_MUTANT value compiles a copy of the oracle with one planted error
(a dropped bias term, a flipped distance sign, the sink left out of the
denominator, an inclusive window bound, a wrong GQA head mapping, a wrong
scale, a sign error in the softmax gradient, an off-by-one dprofiles index,
the query excluded from its own keys, a dropped scale in dk). The pins in
test_oracle.py are run against each copy and at least one must fail.
"""
import contextlib
import os

import pytest

import oracle
from tests import test_oracle as pins

MUTANTS = {
    1: "relative bias dropped",
    2: "distance sign flipped",
    3: "sink left out of the denominator",
    4: "window bound inclusive",
    5: "GQA head mapping interleaved",
    6: "1/D instead of D^-1/2",
    7: "softmax-gradient sign",
    8: "dprofiles index off by one",
    9: "query excluded from its own keys",
    10: "scale dropped in dk",
}

BATTERY = [
    pins.test_tiny_closed_form_forward,
    pins.test_tiny_closed_form_no_bias_beyond_extent,
    pins.test_tiny_closed_form_backward,
    lambda: pins.test_matches_sdpa_with_materialised_bias_and_sink(pins.SHAPES[1]),
    lambda: pins.test_matches_sdpa_with_materialised_bias_and_sink(pins.SHAPES[3]),
    lambda: pins.test_backward_matches_autograd(pins.SHAPES[1], True),
    pins.test_window_bound_readings_differ_by_one_key,
]


@contextlib.contextmanager
def _using(lib):
    saved = oracle._lib
    oracle._lib = lib
    try:
        yield
    finally:
        oracle._lib = saved


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_planted_mistake(mutant, tmp_path):
    path = os.path.join(str(tmp_path), f"liboracle_mutant{mutant}.so")
    oracle.build(out_path=path, defines=(f"ORACLE_MUTANT={mutant}",))
    lib = oracle.load(path)
    failures = 0
    with _using(lib):
        for check in BATTERY:
            try:
                check()
            except AssertionError:
                failures += 1
    assert failures > 0, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"


def test_unmutated_oracle_passes_battery():
    for check in BATTERY:
        check()
