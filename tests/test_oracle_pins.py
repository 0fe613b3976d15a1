"""The CPU oracle against its pins (no GPU).  See tests/oracle_pins.py for what each pin ties
the oracle to and which passage of the pages it follows."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(oracle, pin):
    pin(oracle)


def test_golden_pair_counts_follow_closed_form():
    # The stored counts themselves must equal the FLOPs-table closed form (L^2 + L S) / 2.
    for L, S, pairs in oracle_pins.read_golden_pairs():
        assert pairs == (L * L + L * S) // 2
