"""Pins for the gradient oracle (oracle/sa_backward.py): the gradients of
one SA layer, section 2.1's forward with section 2.2's end-to-end training
("SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模").

Facts used, none of them the backward formulas themselves:
  * central finite differences of the FORWARD oracle (sa_user) in fp64, on
    a scalar loss L = <G, X~> + <g, m> -- the definition of the gradient;
  * k = 1: A == 1, so X~ = column sum, m = n; dX_i = G for every row and
    the prototype and projection gradients vanish;
  * W_Q = 0: S == 0 for any P, so dP = 0 (while dW_Q need not be);
  * a loss on m alone: sum_j m_j = n for any parameters, so a g that is the
    same for every prototype has zero gradient everywhere;
  * the batch form is the per-user form (per-user rows, sums for shared
    weights).
A planted mistake in the backward (a wrong softmax-axis correction, a
missing transpose, a dropped mass term) trips at least one pin."""

import numpy as np
import pytest

from oracle import sa_user
from oracle.sa_backward import sa_batch_backward, sa_user_backward


def _loss(Xb, P, W_Q, W_K, scale, G, g):
    Xt, m = sa_user(Xb, P, W_Q, W_K, scale)
    return float((Xt * G).sum() + (m * g).sum())


def _fd(f, x, eps=1e-6):
    """Central differences of scalar f at array x (x is modified in place
    and restored)."""
    out = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        x0 = x[i]
        x[i] = x0 + eps
        fp = f()
        x[i] = x0 - eps
        fm = f()
        x[i] = x0
        out[i] = (fp - fm) / (2 * eps)
    return out


def _case(seed, n=7, k=4, d=5, scale=0.6):
    rng = np.random.default_rng(seed)
    return dict(Xb=rng.standard_normal((n, d)), P=rng.standard_normal((k, d)),
                W_Q=rng.standard_normal((d, d)) / np.sqrt(d),
                W_K=rng.standard_normal((d, d)) / np.sqrt(d), scale=scale,
                G=rng.standard_normal((k, d)), g=rng.standard_normal(k))


def pin_finite_differences(bwd=sa_user_backward):
    for seed in (1, 2, 3):
        c = _case(seed)
        r = bwd(c["Xb"], c["P"], c["W_Q"], c["W_K"], c["scale"], c["G"], c["g"])
        for name, key in (("dX", "Xb"), ("dP", "P"), ("dW_Q", "W_Q"), ("dW_K", "W_K")):
            arr = c[key]
            fd = _fd(lambda: _loss(c["Xb"], c["P"], c["W_Q"], c["W_K"], c["scale"], c["G"],
                                   c["g"]), arr)
            np.testing.assert_allclose(r[name], fd, rtol=1e-6, atol=1e-8,
                                       err_msg=f"{name} seed {seed}")


def pin_k1_closed_form(bwd=sa_user_backward):
    c = _case(4, k=1)
    r = bwd(c["Xb"], c["P"], c["W_Q"], c["W_K"], c["scale"], c["G"], c["g"])
    np.testing.assert_allclose(r["dX"], np.repeat(c["G"], c["Xb"].shape[0], axis=0), atol=1e-12)
    for name in ("dP", "dW_Q", "dW_K"):
        np.testing.assert_allclose(r[name], 0.0, atol=1e-12, err_msg=name)


def pin_zero_query_projection(bwd=sa_user_backward):
    c = _case(5)
    r = bwd(c["Xb"], c["P"], np.zeros_like(c["W_Q"]), c["W_K"], c["scale"], c["G"], c["g"])
    np.testing.assert_allclose(r["dP"], 0.0, atol=1e-12)
    assert np.abs(r["dW_Q"]).max() > 1e-3


def pin_uniform_mass_loss(bwd=sa_user_backward):
    c = _case(6)
    g = np.full(c["P"].shape[0], 0.7)
    r = bwd(c["Xb"], c["P"], c["W_Q"], c["W_K"], c["scale"], np.zeros_like(c["G"]), g)
    for name in ("dX", "dP", "dW_Q", "dW_K"):
        np.testing.assert_allclose(r[name], 0.0, atol=1e-12, err_msg=name)


PINS = [pin_finite_differences, pin_k1_closed_form, pin_zero_query_projection,
        pin_uniform_mass_loss]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_backward_oracle_satisfies_pin(pin):
    pin()


def test_batch_is_per_user():
    rng = np.random.default_rng(9)
    lens = [5, 0, 3, 6]
    offs = np.concatenate([[0], np.cumsum(lens)])
    d, k = 4, 3
    X = rng.standard_normal((offs[-1], d))
    P = rng.standard_normal((k, d))
    W_Q, W_K = rng.standard_normal((d, d)), rng.standard_normal((d, d))
    G = rng.standard_normal((len(lens), k, d))
    g = rng.standard_normal((len(lens), k))
    Q = rng.standard_normal((len(lens), k, d))
    for queries in (None, Q):
        r = sa_batch_backward(X, offs, P, W_Q, W_K, 0.5, G, g, queries=queries)
        dWQ = np.zeros((d, d))
        dWK = np.zeros((d, d))
        for b in range(len(lens)):
            Pb = P if queries is None else queries[b]
            u = sa_user_backward(X[offs[b]:offs[b + 1]], Pb, W_Q, W_K, 0.5, G[b], g[b])
            np.testing.assert_allclose(r["dX"][offs[b]:offs[b + 1]], u["dX"], atol=1e-12)
            if queries is not None:
                np.testing.assert_allclose(r["dQueries"][b], u["dP"], atol=1e-12)
            dWQ += u["dW_Q"]
            dWK += u["dW_K"]
        np.testing.assert_allclose(r["dW_Q"], dWQ, atol=1e-12)
        np.testing.assert_allclose(r["dW_K"], dWK, atol=1e-12)
    assert np.all(r["dQueries"][1] == 0)  # the empty user


def _mutant(kind):
    """A planted mistake in a copy of the backward."""
    def bwd(Xb, P, W_Q, W_K, scale, G, g=None):
        Xb, P, W_Q, W_K, G = (np.asarray(a, np.float64) for a in (Xb, P, W_Q, W_K, G))
        k, d = P.shape
        g = np.zeros(k) if g is None else np.asarray(g, np.float64)
        K = Xb @ W_K
        Q = P @ W_Q
        S = (Q @ K.T) * scale
        E = np.exp(S - S.max(axis=0, keepdims=True))
        A = E / E.sum(axis=0, keepdims=True)
        dA = G @ Xb.T + (0.0 if kind == "no_mass" else g[:, None])
        axis = 1 if kind == "axis" else 0
        dS = A * (dA - (A * dA).sum(axis=axis, keepdims=True))
        dQ = scale * (dS @ K)
        dK = scale * (dS.T @ Q)
        dX = A.T @ G + (dK @ W_K if kind == "transpose" else dK @ W_K.T)
        return dict(dX=dX, dP=dQ @ W_Q.T, dW_Q=P.T @ dQ, dW_K=Xb.T @ dK)
    return bwd


@pytest.mark.parametrize("kind", ["axis", "transpose", "no_mass"])
def test_a_planted_mistake_trips_a_pin(kind):
    tripped = 0
    for pin in PINS:
        try:
            pin(_mutant(kind))
        except AssertionError:
            tripped += 1
    assert tripped >= 1


def test_q_prime_form_of_the_gradients():
    # The form a fused backward pass computes (S = X Q'^T with
    # Q' = P W_Q W_K^T scale, and the per-user accumulator R = dS X):
    #   dX = A^T G + dS^T Q',  dP = scale R W_K W_Q^T,
    #   dW_Q = scale P^T R W_K,  dW_K = scale R^T P W_Q
    # equals the oracle's chain rule through K = X W_K and Q = P W_Q.
    c = _case(11, n=9, k=5, d=6)
    X, P, WQ, WK, sc, G, g = (c[key] for key in ("Xb", "P", "W_Q", "W_K", "scale", "G", "g"))
    Qp = P @ WQ @ WK.T * sc
    S = Qp @ X.T
    E = np.exp(S - S.max(axis=0, keepdims=True))
    A = E / E.sum(axis=0, keepdims=True)
    dA = G @ X.T + g[:, None]
    dS = A * (dA - (A * dA).sum(axis=0, keepdims=True))
    R = dS @ X
    r = sa_user_backward(X, P, WQ, WK, sc, G, g)
    np.testing.assert_allclose(A.T @ G + dS.T @ Qp, r["dX"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sc * R @ WK @ WQ.T, r["dP"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sc * P.T @ R @ WK, r["dW_Q"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sc * R.T @ P @ WQ, r["dW_K"], rtol=1e-12, atol=1e-12)
