"""Planted mistakes in the oracle must each trip at least one pin.

Mistakes (see kda_oracle.c): 1 state decay dropped, 2 wrong sign in the delta
correction, 3 output read before the update, 4 transposed state in the output,
5 diagonal dropped from the q.k mask, 6 carry-over state not decayed,
7 dt_bias sign, 9 missing square root in the normalise, 10 beta sigmoid dropped;
in the chunked form: 11 the key-key product transposed (K- K~^T for K~ K-^T),
12 W built from K- instead of K~, 13 the chunk's decay taken at its first row instead
of its last, 14 the identity term dropped from the forward substitution, 15 beta
missing from U, 16 the state transposed in Delta; 17 the sign of A_log in the gate.
"""
import pytest

import oracle
import oracle_pins as P

MUTATIONS = [1, 2, 3, 4, 5, 6, 7, 9, 10, 11, 12, 13, 14, 15, 16, 17]


@pytest.mark.parametrize("m", MUTATIONS)
def test_mutation_is_caught(m):
    failed = []
    oracle.set_mutation(m)
    try:
        for pin in P.ALL_PINS:
            try:
                pin()
            except AssertionError:
                failed.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert failed, f"mutation {m} slipped through every pin"


def test_oracle_restored_after_mutations():
    oracle.set_mutation(0)
    P.pin_brute_force_tiny()
