"""Pins for the action-fusion oracle (oracle/sa_action.py).

What the notes' section 2.2 fixes (the formula itself was lost): x_i is e_i
plus a SwiGLU-gated FFN of the concatenation [e_i ; a_i] mapped back to the
item width; the action type changes what the same video means.  The pins
are hand-worked cases whose values follow from SiLU(ln 3) = (3/4) ln 3 and
SiLU(-ln 3) = -(1/4) ln 3 (sigma(ln 3) = 3/4), plus invariants:

* W_2 = 0 leaves x = e exactly (the residual);
* a one-unit network where the gate reads e_0 and the value reads a: the
  residual, the gate branch, the concatenation order and the type lookup
  each change the answer;
* a two-unit network with an asymmetric W_2: the sum over hidden units and
  the orientation of W_2 (h x d) each change the answer;
* rows are independent: the same (e, type) gives the same x wherever it
  sits, a different type gives a different x.

Planted mistakes (each trips a pin): no residual, SiLU on the value branch,
[a ; e] order, a sigmoid in place of SiLU, the type ignored, W_2 read
transposed.
"""

import math

import numpy as np
import pytest

from oracle.sa_action import action_fuse

L3 = math.log(3.0)


def pin_residual_only(fuse=action_fuse):
    rng = np.random.default_rng(0)
    E = rng.standard_normal((5, 4))
    W1, W3 = rng.standard_normal((6, 3)), rng.standard_normal((6, 3))
    X = fuse(E, [0, 1, 2, 1, 0], rng.standard_normal((3, 2)), W1, W3, np.zeros((3, 4)))
    assert np.array_equal(X, E)


def pin_one_unit(fuse=action_fuse):
    E = np.array([[L3, 5.0], [0.0, 1.0], [L3, 5.0]])
    table = np.array([[2.0], [-1.0]])
    W1 = np.array([[1.0], [0.0], [0.0]])   # gate input u = e_0
    W3 = np.array([[0.0], [0.0], [1.0]])   # value v = a
    W2 = np.array([[1.0, 0.0]])
    X = fuse(E, [0, 0, 1], table, W1, W3, W2)
    want = np.array([[2.5 * L3, 5.0], [0.0, 1.0], [0.25 * L3, 5.0]])
    assert np.max(np.abs(X - want)) < 1e-14


def pin_two_units(fuse=action_fuse):
    E = np.array([[L3, -L3]])
    table = np.array([[4.0]])
    W1 = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]])   # u = e
    W3 = np.array([[0.0, 0.0], [0.0, 0.0], [1.0, 1.0]])   # v = (a, a)
    W2 = np.array([[0.0, 2.0], [1.0, 0.0]])
    # g = (SiLU(ln 3) * 4, SiLU(-ln 3) * 4) = (3 ln 3, -ln 3); g W2 = (-ln 3, 6 ln 3)
    X = fuse(E, [0], table, W1, W3, W2)
    assert np.max(np.abs(X - np.array([[0.0, 5.0 * L3]]))) < 1e-14


def pin_rows_independent(fuse=action_fuse):
    rng = np.random.default_rng(1)
    d, da, h = 4, 3, 5
    e = rng.standard_normal(d)
    E = np.stack([e, rng.standard_normal(d), e, e])
    table = rng.standard_normal((3, da))
    W1, W3 = rng.standard_normal((d + da, h)), rng.standard_normal((d + da, h))
    W2 = rng.standard_normal((h, d))
    X = fuse(E, [2, 0, 2, 1], table, W1, W3, W2)
    assert np.array_equal(X[0], X[2])
    assert np.max(np.abs(X[0] - X[3])) > 1e-3
    Xp = fuse(E[::-1], [1, 2, 0, 2], table, W1, W3, W2)
    assert np.array_equal(Xp, X[::-1])


PINS = [pin_residual_only, pin_one_unit, pin_two_units, pin_rows_independent]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_action_oracle_satisfies_pin(pin):
    pin()


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _concat(E, types, table, a_first=False):
    A = np.asarray(table, float)[np.asarray(types)]
    return np.concatenate([A, E] if a_first else [E, A], axis=-1)


MUTANTS = {
    "no residual": lambda E, t, T, W1, W3, W2:
        (lambda Z: (Z @ W1 * _sig(Z @ W1) * (Z @ W3)) @ W2)(_concat(E, t, T)),
    "SiLU on the value branch": lambda E, t, T, W1, W3, W2:
        E + (lambda Z: ((Z @ W1) * (Z @ W3) * _sig(Z @ W3)) @ W2)(_concat(E, t, T)),
    "[a ; e] order": lambda E, t, T, W1, W3, W2:
        E + (lambda Z: (Z @ W1 * _sig(Z @ W1) * (Z @ W3)) @ W2)(_concat(E, t, T, a_first=True)),
    "sigmoid for SiLU": lambda E, t, T, W1, W3, W2:
        E + (lambda Z: (_sig(Z @ W1) * (Z @ W3)) @ W2)(_concat(E, t, T)),
    "type ignored": lambda E, t, T, W1, W3, W2:
        E + (lambda Z: (Z @ W1 * _sig(Z @ W1) * (Z @ W3)) @ W2)(_concat(E, np.zeros_like(t), T)),
    "W2 transposed": lambda E, t, T, W1, W3, W2:
        E + (lambda Z: (Z @ W1 * _sig(Z @ W1) * (Z @ W3)) @ np.asarray(W2).T)(_concat(E, t, T)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_action_mutant_is_caught(name):
    caught = []
    for pin in PINS:
        try:
            pin(fuse=MUTANTS[name])
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name!r} passed every pin"
