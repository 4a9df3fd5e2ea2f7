"""The oracle against its pins (closed forms, special cases, brute force, invariants)."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin()


def test_chunked_equals_recurrent_lower_bound_zero():
    # lower_bound = 0 path: no decay, long memory
    P.pin_chunked_equals_recurrent(seed=11, lb=0.0, Ls=(3, 70), Cs=(1, 64))


hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402
import numpy as np  # noqa: E402

import oracle  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(L=st.integers(1, 150), C=st.integers(1, 70), Dk=st.integers(1, 12), Dv=st.integers(1, 12),
       lb=st.floats(-5.0, 0.0), seed=st.integers(0, 2**31 - 1))
def test_chunked_equals_recurrent_random_shapes(L, C, Dk, Dv, lb, seed):
    """Invariant I1 over random lengths, chunk sizes (tails of every size), head dims and gate
    bounds: the chunked form reaches the token recurrence's outputs and final state."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = P._rand_unit_inputs(rng, L, Dk, Dv, lb)
    o_r, S_r = oracle.recurrent(q, k, v, g, beta, 0.3, S0)
    o_c, S_c = oracle.chunked(q, k, v, g, beta, 0.3, S0, C=C)
    assert P._rel(o_c, o_r) < 1e-9 and P._rel(S_c, S_r) < 1e-9
