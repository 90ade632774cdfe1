"""Pins for the CPU oracle: checks against facts fixed by the method's
definition and by mathematics, not against the oracle itself.

Each ``pin_*`` function takes ``steps`` (oracle step overrides, default none)
and raises AssertionError when the oracle built from those steps violates the
pinned fact.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` plants plausible mistakes in the oracle and checks
that each one trips at least one pin.

Facts used (SequenceO1 reading notes, "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模"):
  * section 2.1: the normaliser sums over prototypes, so every behaviour's
    weights sum to one  =>  sum_j m_j = n for every user;
  * section 2.1: X itself is aggregated (no value projection)  =>  with k = 1
    the sketch is the column sum of X and m = n;
  * section 2.1: weighted aggregation, order not kept  =>  invariance under a
    permutation of a user's rows; prototypes are only labels  =>
    equivariance under a permutation of P's rows;
  * section 2.4: stable softmax statistics  =>  finite results at logits of
    order 1e4;
  * section 3.1: padding must not receive mass  =>  rows outside a user's
    range (even NaN) do not change its outputs;
  * mathematics: the 2-prototype softmax is a logistic function (closed form);
    linearity in the rows (additivity, doubling); identical prototypes give
    A = 1/k; a common shift of all prototypes by c leaves A unchanged; the
    large-scale limit is the hard argmax assignment (the k-means assignment
    sum); and a pure-Python brute force on tiny inputs.
"""

from __future__ import annotations

import math

import numpy as np

from oracle import sa_batch, sa_user, sa_user_bruteforce


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _inputs(rng, n, k, d, scale=None):
    X = _rand(rng, n, d)
    P = _rand(rng, k, d)
    W_Q = _rand(rng, d, d) / math.sqrt(d)
    W_K = _rand(rng, d, d) / math.sqrt(d)
    return X, P, W_Q, W_K, (1.0 / math.sqrt(d)) if scale is None else scale


def _close(a, b, rtol, atol=0.0, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    ref = max(np.max(np.abs(b)) if b.size else 0.0, 1e-300)
    assert err <= rtol * ref + atol, f"{what}: max err {err:.3e} > {rtol:.1e} * {ref:.3e}"


# ---------------------------------------------------------------------------

def pin_bruteforce(steps=None):
    """Tiny random inputs: oracle == pure-Python loops, to 1e-12."""
    rng = np.random.default_rng(7)
    for n, k, d in [(1, 1, 1), (3, 2, 2), (5, 3, 4), (8, 4, 3), (6, 4, 4)]:
        X, P, W_Q, W_K, scale = _inputs(rng, n, k, d, scale=0.7)
        Xt, m = sa_user(X, P, W_Q, W_K, scale, steps=steps)
        bXt, bm = sa_user_bruteforce(X.tolist(), P.tolist(), W_Q.tolist(),
                                     W_K.tolist(), scale)
        _close(Xt, bXt, 1e-12, 1e-14, "brute X~")
        _close(m, bm, 1e-12, 1e-14, "brute m")


def pin_two_prototype_logistic(steps=None):
    """k = 2, d = 1, W_Q = W_K = [[1]], P = [[a], [b]]:
    S_ji = scale * p_j * x_i and A_0i = 1 / (1 + exp(scale (b - a) x_i))."""
    a, b, scale = 1.25, -0.5, 0.8
    xs = [0.5, -1.0, 2.0, 0.0, -3.5]
    A0 = [1.0 / (1.0 + math.exp(scale * (b - a) * x)) for x in xs]
    want_Xt = [[sum(p * x for p, x in zip(A0, xs))],
               [sum((1.0 - p) * x for p, x in zip(A0, xs))]]
    want_m = [sum(A0), len(xs) - sum(A0)]
    Xt, m = sa_user(np.array(xs)[:, None], np.array([[a], [b]]), np.eye(1),
                    np.eye(1), scale, steps=steps)
    _close(Xt, want_Xt, 1e-13, 1e-15, "logistic X~")
    _close(m, want_m, 1e-13, 1e-15, "logistic m")


def pin_total_mass_is_n(steps=None):
    """sum_j m_j == n_b for every user, including large logits."""
    rng = np.random.default_rng(11)
    for n, k, d, s in [(1, 5, 3, None), (37, 7, 8, None), (200, 16, 16, 40.0)]:
        X, P, W_Q, W_K, scale = _inputs(rng, n, k, d, s)
        Xt, m = sa_user(X, P, W_Q, W_K, scale, steps=steps)
        assert m.shape == (k,), f"mass shape {m.shape}"
        assert abs(m.sum() - n) <= 1e-12 * n, f"sum m = {m.sum()} != n = {n}"
        assert np.all(m >= 0), "negative mass"


def pin_k1_column_sum(steps=None):
    """k = 1: every weight is 1, so X~ = sum_i x_i and m = n (no value
    projection)."""
    rng = np.random.default_rng(13)
    X, P, W_Q, W_K, scale = _inputs(rng, 50, 1, 6)
    Xt, m = sa_user(X, P, W_Q, W_K, scale, steps=steps)
    _close(Xt, X.sum(axis=0, keepdims=True), 1e-13, 0, "k=1 X~")
    _close(m, [50.0], 1e-14, 0, "k=1 m")


def pin_uniform_assignment(steps=None):
    """Identical prototypes, W_Q = 0 or W_K = 0: A = 1/k, so X~_j = sum X / k
    and m_j = n / k."""
    rng = np.random.default_rng(17)
    n, k, d = 40, 6, 5
    X, P, W_Q, W_K, scale = _inputs(rng, n, k, d)
    want_Xt = np.tile(X.sum(axis=0) / k, (k, 1))
    want_m = np.full(k, n / k)
    cases = [(np.tile(P[:1], (k, 1)), W_Q, W_K),
             (P, np.zeros((d, d)), W_K),
             (P, W_Q, np.zeros((d, d)))]
    for Pc, WQc, WKc in cases:
        Xt, m = sa_user(X, Pc, WQc, WKc, scale, steps=steps)
        _close(Xt, want_Xt, 1e-12, 0, "uniform X~")
        _close(m, want_m, 1e-12, 0, "uniform m")


def pin_prototype_shift(steps=None):
    """P -> P + 1 c^T adds the same amount to every prototype's logit for a
    given behaviour, which the softmax over prototypes cancels."""
    rng = np.random.default_rng(19)
    X, P, W_Q, W_K, scale = _inputs(rng, 30, 5, 4)
    c = rng.standard_normal(4) * 3.0
    a = sa_user(X, P, W_Q, W_K, scale, steps=steps)
    b = sa_user(X, P + c[None, :], W_Q, W_K, scale, steps=steps)
    _close(b[0], a[0], 1e-10, 0, "shift X~")
    _close(b[1], a[1], 1e-10, 0, "shift m")


def pin_permutations(steps=None):
    """Row permutation inside a user: outputs unchanged.  Prototype
    permutation: output rows permuted the same way."""
    rng = np.random.default_rng(23)
    X, P, W_Q, W_K, scale = _inputs(rng, 33, 6, 5)
    Xt, m = sa_user(X, P, W_Q, W_K, scale, steps=steps)
    pr = rng.permutation(33)
    Xt2, m2 = sa_user(X[pr], P, W_Q, W_K, scale, steps=steps)
    _close(Xt2, Xt, 1e-12, 0, "row perm X~")
    _close(m2, m, 1e-12, 0, "row perm m")
    pj = rng.permutation(6)
    Xt3, m3 = sa_user(X, P[pj], W_Q, W_K, scale, steps=steps)
    _close(Xt3, Xt[pj], 1e-12, 0, "proto perm X~")
    _close(m3, m[pj], 1e-12, 0, "proto perm m")


def pin_additivity(steps=None):
    """Columns are independent: X~(X) = X~(X[:t]) + X~(X[t:]); duplicating
    every row doubles X~ and m."""
    rng = np.random.default_rng(29)
    X, P, W_Q, W_K, scale = _inputs(rng, 41, 5, 6)
    full = sa_user(X, P, W_Q, W_K, scale, steps=steps)
    for t in (1, 17, 40):
        a = sa_user(X[:t], P, W_Q, W_K, scale, steps=steps)
        b = sa_user(X[t:], P, W_Q, W_K, scale, steps=steps)
        _close(a[0] + b[0], full[0], 1e-12, 0, "split X~")
        _close(a[1] + b[1], full[1], 1e-12, 0, "split m")
    dbl = sa_user(np.concatenate([X, X]), P, W_Q, W_K, scale, steps=steps)
    _close(dbl[0], 2 * full[0], 1e-12, 0, "double X~")
    _close(dbl[1], 2 * full[1], 1e-12, 0, "double m")


def pin_hard_assignment_limit(steps=None):
    """With a very large scale the weights become one-hot on each behaviour's
    best prototype, and X~_j becomes the k-means assignment sum over the
    behaviours assigned to j.  Logits reach ~1e4 here, which the stable
    softmax must survive.  The argmax is taken on the reassociated logits
    x_i (W_K W_Q^T p_j), a different evaluation order from the oracle's."""
    rng = np.random.default_rng(31)
    n, k, d = 300, 7, 8
    X, P, W_Q, W_K, _ = _inputs(rng, n, k, d)
    scale = 5e3
    logits = X @ (W_K @ (W_Q.T @ P.T))  # (n, k), unscaled
    top2 = np.sort(logits, axis=1)[:, -2:]
    keep = (top2[:, 1] - top2[:, 0]) > 0.02  # drop near-ties
    X, logits = X[keep], logits[keep]
    assign = np.argmax(logits, axis=1)
    want_Xt = np.zeros((k, d))
    np.add.at(want_Xt, assign, X)
    want_m = np.bincount(assign, minlength=k).astype(np.float64)
    Xt, m = sa_user(X, P, W_Q, W_K, scale, steps=steps)
    assert np.max(np.abs(logits * scale)) > 1e3
    _close(Xt, want_Xt, 1e-9, 1e-9, "hard X~")
    _close(m, want_m, 1e-9, 1e-9, "hard m")


def pin_batch_isolation(steps=None):
    """Ragged batch: each user sees only its own rows.  NaN / huge rows in the
    neighbours (and empty users) must not leak into a user's outputs."""
    rng = np.random.default_rng(37)
    d, k = 4, 3
    lens = [5, 0, 9, 1, 0, 7]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    X = rng.standard_normal((offs[-1], d))
    _, P, W_Q, W_K, scale = _inputs(rng, 1, k, d)
    Xt, m = sa_batch(X, offs, P, W_Q, W_K, scale, steps=steps)
    for b, (lo, hi) in enumerate(zip(offs[:-1], offs[1:])):
        if hi == lo:
            assert np.all(Xt[b] == 0) and np.all(m[b] == 0), "empty user not zero"
            continue
        Xb_t, mb = sa_user(X[lo:hi], P, W_Q, W_K, scale, steps=steps)
        _close(Xt[b], Xb_t, 0, 0, f"user {b} X~")
        _close(m[b], mb, 0, 0, f"user {b} m")
    poisoned = X.copy()
    poisoned[offs[2]:offs[3]] = np.nan  # user 2's rows
    poisoned[offs[5]:offs[6]] = 1e30
    Xt2, m2 = sa_batch(poisoned, offs, P, W_Q, W_K, scale, users=[0, 3],
                       steps=steps)
    for b in (0, 3):
        _close(Xt2[b], Xt[b], 0, 0, f"poisoned neighbours X~ user {b}")
        _close(m2[b], m[b], 0, 0, f"poisoned neighbours m user {b}")


ALL_PINS = [
    pin_bruteforce,
    pin_two_prototype_logistic,
    pin_total_mass_is_n,
    pin_k1_column_sum,
    pin_uniform_assignment,
    pin_prototype_shift,
    pin_permutations,
    pin_additivity,
    pin_hard_assignment_limit,
    pin_batch_isolation,
]
