"""The oracle against its pins (closed forms, special cases, brute force, invariants)."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin()


def test_chunked_equals_recurrent_lower_bound_zero():
    # lower_bound = 0 path: no decay, long memory
    P.pin_chunked_equals_recurrent(seed=11, lb=0.0, Ls=(3, 70), Cs=(1, 64))
