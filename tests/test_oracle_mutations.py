"""Planted mistakes in the oracle must be caught by the pins.

Each mutation is a plausible slip named in the pages' own bug reports (ALiBi
before softcap, NaN turned into 0, an unguarded exp(-inf - -inf) on an empty
row, a narrowed F16 mask -- HartsyInference PR #910; duplicate or invalid
selection entries not skipped -- strix-llama.cpp PR #115/#119) or a generic one
(wrong sign, wrong GQA index, reversed operand, off-by-one causality), or a
slip in the dequantization of an e4m3 / int8 cache (wrong exponent bias, the
NaN code read as a number, a scale taken from the wrong cell, head or tensor,
int8 read unsigned).  The mistake is planted in the oracle, on the CPU, and the
pin suite must go red.
"""
import pytest

import oracle
import oracle_pins


def _failing_pins():
    failed = []
    for name, fn in sorted(oracle_pins.PINS.items()):
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


@pytest.mark.parametrize("mutation", sorted(oracle.MUTATIONS))
def test_pins_catch_mutation(mutation):
    with oracle.mutation(mutation):
        failed = _failing_pins()
    assert failed, f"no pin catches the planted mistake '{mutation}'"
