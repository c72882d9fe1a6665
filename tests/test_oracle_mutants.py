"""Every planted mistake in the oracle must turn at least one pin red (CPU only).

The mistakes are compiled into separate copies of the oracle (CKDA_ORACLE_MUTANT=n); the real
oracle is never modified.  This shows the pins in pins.py can see each class of error: the order
of Diag(alpha) and the rank-one factor, the gate sign, the beta range, the read-out state, the
read-out scale, the rotary frequency, rotating only q, the rotary base, a missing L2 norm and a
norm taken jointly over q and k, and the two gate activations.
"""
import pytest

import oracle
import pins

MUTANTS = {
    1: "Diag(alpha) applied after the rank-one factor",
    2: "sign of alpha dropped",
    3: "beta clamped to 1",
    4: "output read from S_{t-1}",
    5: "read-out scale dropped",
    6: "rotary frequency without its factor 2",
    7: "rotation applied to q only",
    8: "rotary base 1000",
    9: "L2 norm skipped",
    10: "L2 norm over q and k jointly",
    11: "signed gate as sigma(a), without the 2x - 1 map",
    12: "beta as sigma(b), without the factor 2",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: f"mut{m}")
def test_mutant_is_caught(mutant):
    assert oracle.mutant_id(mutant) == mutant
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant=mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {mutant}: {MUTANTS[mutant]}"


def test_real_oracle_is_not_a_mutant():
    assert oracle.mutant_id(0) == 0
