"""Pins for the oracle's mass-normalised sketch, oracle.mass_normalised.

X~_j / m_j is the weighted mean of a user's rows under prototype j (section
2.1 of the SequenceO1 reading notes: the sketch is a weighted aggregation of
the rows, every behaviour spreading unit weight over the prototypes; the
mass m_j is that weight summed over the behaviours).  Each pin checks it
against a fact that does not come from the oracle:

  * identical prototypes give A = 1/k, so every X~_j / m_j is the plain mean
    of the user's rows (numpy's mean);
  * k = 1 gives the column mean for any weights;
  * the hard-assignment limit gives the k-means centroid of the rows
    assigned to prototype j (argmax on the reassociated logits);
  * a weighted mean lies inside the range of the rows, feature by feature;
  * m_j == 0 gives exactly 0, never NaN or inf (reading R4);
  * the normalisation is per prototype and per user: scaling one user's
    sketch row and mass by the same factor leaves every output unchanged.

Two planted mistakes (dividing by the user's total mass, i.e. the wrong
axis of m; and plain division, which gives NaN at m = 0) each trip a pin.
"""

import math

import numpy as np
import pytest

from oracle import mass_normalised, sa_batch, sa_user


def _inputs(rng, n, k, d):
    X = rng.standard_normal((n, d))
    P = rng.standard_normal((k, d))
    W_Q = rng.standard_normal((d, d)) / math.sqrt(d)
    W_K = rng.standard_normal((d, d)) / math.sqrt(d)
    return X, P, W_Q, W_K, 1.0 / math.sqrt(d)


def pin_identical_prototypes_give_row_mean(fn=mass_normalised):
    rng = np.random.default_rng(41)
    n, k, d = 57, 5, 6
    X, P, W_Q, W_K, scale = _inputs(rng, n, k, d)
    Pc = np.tile(P[:1], (k, 1))
    Xt, m = sa_user(X, Pc, W_Q, W_K, scale)
    got = fn(Xt, m)
    want = np.tile(X.mean(axis=0), (k, 1))
    assert got.shape == (k, d)
    assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


def pin_k1_is_column_mean(fn=mass_normalised):
    rng = np.random.default_rng(43)
    X, P, W_Q, W_K, scale = _inputs(rng, 33, 1, 7)
    Xt, m = sa_user(X, P, W_Q, W_K, scale)
    got = fn(Xt, m)
    assert np.max(np.abs(got[0] - X.mean(axis=0))) <= 1e-13


def pin_hard_assignment_gives_centroids(fn=mass_normalised):
    rng = np.random.default_rng(47)
    n, k, d = 400, 6, 8
    X, P, W_Q, W_K, _ = _inputs(rng, n, k, d)
    logits = X @ (W_K @ (W_Q.T @ P.T))
    top2 = np.sort(logits, axis=1)[:, -2:]
    keep = (top2[:, 1] - top2[:, 0]) > 0.02
    X, logits = X[keep], logits[keep]
    assign = np.argmax(logits, axis=1)
    Xt, m = sa_user(X, P, W_Q, W_K, 5e3)
    got = fn(Xt, m)
    for j in range(k):
        rows = X[assign == j]
        if len(rows) == 0:
            assert np.all(got[j] == 0.0)
        else:
            assert np.max(np.abs(got[j] - rows.mean(axis=0))) <= 1e-9


def pin_inside_row_range(fn=mass_normalised):
    rng = np.random.default_rng(53)
    X, P, W_Q, W_K, scale = _inputs(rng, 25, 9, 5)
    Xt, m = sa_user(X, P, W_Q, W_K, 3.0)
    got = fn(Xt, m)
    lo, hi = X.min(axis=0), X.max(axis=0)
    assert np.all(got >= lo - 1e-12) and np.all(got <= hi + 1e-12)


def pin_zero_mass_gives_zero(fn=mass_normalised):
    """Batch with an empty user (m = 0 everywhere) and a prototype whose mass
    is set to 0 by hand: those rows are exactly 0, the others unchanged."""
    rng = np.random.default_rng(59)
    d, k = 4, 3
    lens = [6, 0, 11]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    X = rng.standard_normal((offs[-1], d))
    _, P, W_Q, W_K, scale = _inputs(rng, 1, k, d)
    Xt, m = sa_batch(X, offs, P, W_Q, W_K, scale)
    m = m.copy()
    Xt = Xt.copy()
    m[2, 1] = 0.0
    Xt[2, 1] = 0.0
    with np.errstate(all="ignore"):
        got = fn(Xt, m)
    assert np.all(np.isfinite(got)), "non-finite output at zero mass"
    assert np.all(got[1] == 0.0) and np.all(got[2, 1] == 0.0)
    for b, j in [(0, 0), (0, 2), (2, 0), (2, 2)]:
        lo, hi = offs[b], offs[b + 1]
        Xb, mb = sa_user(X[lo:hi], P, W_Q, W_K, scale)
        assert np.max(np.abs(got[b, j] - Xb[j] / mb[j])) <= 1e-13


def pin_per_prototype_scale_invariance(fn=mass_normalised):
    rng = np.random.default_rng(61)
    X, P, W_Q, W_K, scale = _inputs(rng, 40, 5, 6)
    Xt, m = sa_user(X, P, W_Q, W_K, scale)
    base = fn(Xt[None], m[None])[0]
    f = np.array([1.0, 3.0, 0.25, 7.0, 1.5])
    got = fn((Xt * f[:, None])[None], (m * f)[None])[0]
    assert np.max(np.abs(got - base)) <= 1e-13 * np.max(np.abs(base))


PINS = [pin_identical_prototypes_give_row_mean, pin_k1_is_column_mean,
        pin_hard_assignment_gives_centroids, pin_inside_row_range,
        pin_zero_mass_gives_zero, pin_per_prototype_scale_invariance]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_mass_normalised_satisfies_pin(pin):
    pin()


def _by_total_mass(Xt, m):
    m = np.asarray(m, np.float64)
    tot = m.sum(axis=-1, keepdims=True)
    return np.asarray(Xt, np.float64) / tot[..., None]


def _plain_division(Xt, m):
    return np.asarray(Xt, np.float64) / np.asarray(m, np.float64)[..., None]


MUTANTS = {"divided by the user's total mass (wrong axis)": _by_total_mass,
           "plain division (NaN at zero mass)": _plain_division}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mass_normalised_mutant_is_caught(name):
    fn = MUTANTS[name]
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(fn=fn)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name!r} passed every pin"
