"""Plant plausible mistakes in the oracle (on the CPU) and check that every
one of them trips at least one pin.  This is what makes the pins worth
trusting: a dropped term, a wrong sign or axis, or a transposed operand
cannot slip through."""

import numpy as np
import pytest

from oracle_pins import ALL_PINS


def _softmax_axis1(S):
    c = S.max(axis=1, keepdims=True)
    E = np.exp(S - c)
    return E / E.sum(axis=1, keepdims=True)


def _softmax_unstable(S):
    E = np.exp(S)
    return E / E.sum(axis=0, keepdims=True)


def _softmax_wrong_shift(S):
    c = S.max(axis=1, keepdims=True)  # per-prototype shift: not a softmax of S
    E = np.exp(S - c)
    return E / E.sum(axis=0, keepdims=True)


MUTANTS = {
    "softmax over behaviours (token axis)": dict(prototype_softmax=_softmax_axis1),
    "softmax without max subtraction": dict(prototype_softmax=_softmax_unstable),
    "softmax shifted per prototype": dict(prototype_softmax=_softmax_wrong_shift),
    "W_K transposed": dict(project_keys=lambda Xb, W_K: Xb @ W_K.T),
    "W_Q transposed": dict(project_prototypes=lambda P, W_Q: P @ W_Q.T),
    "scale dropped": dict(affinity=lambda Q, K, s: Q @ K.T),
    "scale applied twice": dict(affinity=lambda Q, K, s: (Q @ K.T) * s * s),
    "affinity sign flipped": dict(affinity=lambda Q, K, s: -(Q @ K.T) * s),
    "value projection added": dict(
        aggregate=lambda A, Xb: A @ (Xb @ np.full((Xb.shape[1],) * 2, 0.3))),
    "rows misaligned in aggregation": dict(aggregate=lambda A, Xb: A @ Xb[::-1]),
    "mass summed over prototypes": dict(prototype_mass=lambda A: A.sum(axis=0)),
    "mass averaged instead of summed": dict(
        prototype_mass=lambda A: A.sum(axis=1) / A.shape[1]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    steps = MUTANTS[name]
    caught = []
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(steps=steps)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name!r} passed every pin"
