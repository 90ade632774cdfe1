"""Pins for the oracle's per-user-query SA (sa_batch_user_queries, the SA step
of a refinement layer: section 2.2 "Stacked Refinement" of the SequenceO1
reading notes, "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模").

Facts used, none of them the oracle itself:
  * a pure-Python brute force (independent derivation) on tiny batches;
  * the hard-assignment limit: when each user's queries single out one
    prototype for that user's rows, all of the user's mass and the column sum
    of its rows land on that prototype, so a query taken from the wrong user
    moves them elsewhere;
  * the normaliser sums over prototypes, so sum_j m_j = n_b for every user;
  * a user's outputs do not depend on another user's queries.
Each pin takes the batch function, so that a planted mistake can be shown to
trip it."""

import math

import numpy as np
import pytest

from oracle import sa_batch_user_queries, sa_user_bruteforce


def _ragged(rng, lens, k, d):
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    X = rng.standard_normal((int(offs[-1]), d))
    queries = rng.standard_normal((len(lens), k, d))
    W_Q = rng.standard_normal((d, d)) / math.sqrt(d)
    W_K = rng.standard_normal((d, d)) / math.sqrt(d)
    return X, offs, queries, W_Q, W_K, 1.0 / math.sqrt(d)


def pin_bruteforce(fn=sa_batch_user_queries):
    rng = np.random.default_rng(5)
    X, offs, queries, W_Q, W_K, scale = _ragged(rng, [3, 0, 5, 1], k=3, d=4)
    Xt, m = fn(X, offs, queries, W_Q, W_K, scale)
    for b in range(len(offs) - 1):
        lo, hi = offs[b], offs[b + 1]
        if hi == lo:
            assert np.all(Xt[b] == 0) and np.all(m[b] == 0)
            continue
        Xt_r, m_r = sa_user_bruteforce(X[lo:hi].tolist(), queries[b].tolist(), W_Q.tolist(),
                                       W_K.tolist(), scale)
        np.testing.assert_allclose(Xt[b], np.array(Xt_r), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(m[b], np.array(m_r), rtol=1e-12, atol=1e-12)


def pin_each_user_uses_its_own_queries(fn=sa_batch_user_queries):
    # d = k = 4 users; user b's rows lie near the unit vector e_b, and its
    # queries put a large weight on prototype b along e_b (W_Q = W_K = I), so
    # the hard assignment sends every row of user b to prototype b.
    k = d = B = 4
    rng = np.random.default_rng(6)
    lens = [7, 3, 5, 2]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    X = np.concatenate([np.eye(d)[b] + 0.01 * rng.standard_normal((lens[b], d))
                        for b in range(B)])
    queries = np.zeros((B, k, d))
    for b in range(B):
        queries[b, b] = 200.0 * np.eye(d)[b]
    Xt, m = fn(X, offs, queries, np.eye(d), np.eye(d), 1.0)
    for b in range(B):
        rows = X[offs[b]:offs[b + 1]]
        want_m = np.zeros(k)
        want_m[b] = lens[b]
        np.testing.assert_allclose(m[b], want_m, atol=1e-6)
        np.testing.assert_allclose(Xt[b, b], rows.sum(axis=0), atol=1e-6)


def pin_total_mass(fn=sa_batch_user_queries):
    rng = np.random.default_rng(7)
    lens = [40, 1, 0, 17]
    X, offs, queries, W_Q, W_K, scale = _ragged(rng, lens, k=6, d=8)
    _, m = fn(X, offs, queries, W_Q, W_K, scale)
    np.testing.assert_allclose(m.sum(axis=1), np.array(lens, float), rtol=1e-12, atol=1e-12)


def pin_isolation_from_other_users_queries(fn=sa_batch_user_queries):
    rng = np.random.default_rng(8)
    X, offs, queries, W_Q, W_K, scale = _ragged(rng, [9, 12, 4], k=5, d=8)
    Xt, m = fn(X, offs, queries, W_Q, W_K, scale)
    q2 = queries.copy()
    q2[1] = rng.standard_normal(q2[1].shape) * 10
    Xt2, m2 = fn(X, offs, q2, W_Q, W_K, scale)
    for b in (0, 2):
        assert np.array_equal(Xt[b], Xt2[b]) and np.array_equal(m[b], m2[b])
    assert not np.allclose(Xt[1], Xt2[1])


PINS = [pin_bruteforce, pin_each_user_uses_its_own_queries, pin_total_mass,
        pin_isolation_from_other_users_queries]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_satisfies_pin(pin):
    pin()


def _wrong_user(X, offsets, queries, W_Q, W_K, scale):
    """A planted mistake: user b is queried with user b+1's queries."""
    B = len(offsets) - 1
    return sa_batch_user_queries(X, offsets, np.roll(queries, -1, axis=0), W_Q, W_K, scale) \
        if B > 1 else sa_batch_user_queries(X, offsets, queries, W_Q, W_K, scale)


def _shared_first(X, offsets, queries, W_Q, W_K, scale):
    """A planted mistake: every user is queried with user 0's queries."""
    return sa_batch_user_queries(X, offsets, np.repeat(queries[:1], len(queries), axis=0),
                                 W_Q, W_K, scale)


@pytest.mark.parametrize("mutant", [_wrong_user, _shared_first], ids=lambda f: f.__name__)
def test_a_planted_mistake_trips_a_pin(mutant):
    tripped = 0
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            tripped += 1
    assert tripped >= 1
