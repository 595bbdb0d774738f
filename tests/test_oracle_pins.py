"""The FP64 oracle against the pages' worked examples, a library routine,
closed forms, brute force and invariants (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("name", sorted(oracle_pins.PINS))
def test_pin(name):
    oracle_pins.PINS[name]()
