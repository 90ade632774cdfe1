"""Pins for the refinement-layer oracle (oracle/sa_refine.py).

Section 2.2 of the SequenceO1 reading notes ("Stacked Refinement"): each layer
queries the original history with the previous sketch, adds the aggregation
to it and normalises, then applies a residual feed-forward network and
normalises again (readings F1-F4 in the oracle's header).  The pins check
the oracle against facts that do not come from it:

  * layer normalisation: a hand-computed vector, a constant row maps to
    beta, zero mean and unit variance (up to eps) for gamma = 1, beta = 0;
  * SiLU and the SwiGLU network: closed values, and pure-Python loops on
    tiny shapes;
  * a whole two-layer stack on tiny inputs against pure-Python loops
    (softmax over prototypes, weighted mean, residuals, norms, FFN);
  * with a zero FFN and W_Q = 0 the assignment is uniform, so every
    prototype's aggregation term is the plain mean of the user's rows;
  * with a huge scale and a zero FFN, the aggregation is the k-means
    centroid of the rows whose best prototype is j;
  * row permutations inside a user leave the stack unchanged, and a
    prototype permutation permutes its output rows.

Planted mistakes (each must trip a pin): LN over the prototype axis, the
input residual dropped, the raw sum in place of the mass-normalised sketch,
SiLU on the linear branch, the FFN residual dropped, no eps in the norm.
"""

import math

import numpy as np
import pytest

from oracle import layer_norm, refine_stack, silu, swiglu_ffn
from oracle.sa_refine import LN_EPS


def _params(rng, d, h, scale=None, zero_ffn=False, zero_wq=False):
    p = dict(
        W_Q=np.zeros((d, d)) if zero_wq else rng.standard_normal((d, d)) / math.sqrt(d),
        W_K=rng.standard_normal((d, d)) / math.sqrt(d),
        scale=1.0 / math.sqrt(d) if scale is None else scale,
        gamma1=1.0 + 0.1 * rng.standard_normal(d), beta1=0.1 * rng.standard_normal(d),
        gamma2=1.0 + 0.1 * rng.standard_normal(d), beta2=0.1 * rng.standard_normal(d),
        W1=rng.standard_normal((d, h)) / math.sqrt(d),
        W3=rng.standard_normal((d, h)) / math.sqrt(d),
        W2=rng.standard_normal((h, d)) / math.sqrt(h))
    if zero_ffn:
        p["W1"] = np.zeros((d, h)); p["W3"] = np.zeros((d, h)); p["W2"] = np.zeros((h, d))
    return p


# ----------------------------------------------------------------- brute force

def _bf_ln(v, g, b):
    n = len(v)
    mu = sum(v) / n
    var = sum((x - mu) ** 2 for x in v) / n
    return [(x - mu) / math.sqrt(var + LN_EPS) * g[i] + b[i] for i, x in enumerate(v)]


def _bf_ffn(z, W1, W3, W2):
    d, h = len(z), len(W1[0])
    a = [sum(z[i] * W1[i][c] for i in range(d)) for c in range(h)]
    g = [sum(z[i] * W3[i][c] for i in range(d)) for c in range(h)]
    u = [a[c] / (1.0 + math.exp(-a[c])) * g[c] for c in range(h)]
    return [sum(u[c] * W2[c][j] for c in range(h)) for j in range(d)]


def _bf_layer(Xb, Q, prev, L):
    """One layer for one user with pure-Python loops: S_ji = scale (q_j W_Q).(x_i W_K),
    softmax over j, weighted mean per prototype, residual + LN, FFN + LN."""
    d = len(Xb[0])
    k = len(Q)
    WQ, WK = L["W_Q"].tolist(), L["W_K"].tolist()
    qp = [[sum(Q[j][a] * WQ[a][c] for a in range(d)) for c in range(d)] for j in range(k)]
    xk = [[sum(x[a] * WK[a][c] for a in range(d)) for c in range(d)] for x in Xb]
    A = [[0.0] * len(Xb) for _ in range(k)]
    for i in range(len(Xb)):
        s = [L["scale"] * sum(qp[j][c] * xk[i][c] for c in range(d)) for j in range(k)]
        mx = max(s)
        e = [math.exp(v - mx) for v in s]
        z = sum(e)
        for j in range(k):
            A[j][i] = e[j] / z
    out = []
    for j in range(k):
        mj = sum(A[j])
        M = [sum(A[j][i] * Xb[i][c] for i in range(len(Xb))) / mj if mj > 0 else 0.0
             for c in range(d)]
        xbar = _bf_ln([prev[j][c] + M[c] for c in range(d)], L["gamma1"].tolist(),
                      L["beta1"].tolist())
        f = _bf_ffn(xbar, L["W1"].tolist(), L["W3"].tolist(), L["W2"].tolist())
        out.append(_bf_ln([xbar[c] + f[c] for c in range(d)], L["gamma2"].tolist(),
                          L["beta2"].tolist()))
    return out


def _bf_stack(X, offsets, P, layers):
    outs = []
    for b in range(len(offsets) - 1):
        Xb = X[offsets[b]:offsets[b + 1]].tolist()
        prev = P.tolist()
        for L in layers:
            prev = _bf_layer(Xb, prev, prev, L) if Xb else None
            if prev is None:
                break
        outs.append(prev)
    return outs


# ----------------------------------------------------------------- pins

def pin_layer_norm(steps=None):
    del steps
    v = np.array([1.0, 2.0, 3.0, 6.0])
    mu, var = 3.0, (4 + 1 + 0 + 9) / 4.0
    want = (v - mu) / math.sqrt(var + LN_EPS)
    got = layer_norm(v, np.ones(4), np.zeros(4))
    assert np.max(np.abs(got - want)) < 1e-14
    g, b = np.array([2.0, -1.0, 0.5, 3.0]), np.array([0.1, 0.2, -0.3, 4.0])
    assert np.max(np.abs(layer_norm(v, g, b) - (want * g + b))) < 1e-14
    assert np.max(np.abs(layer_norm(np.full(4, 7.5), g, b) - b)) < 1e-12
    rng = np.random.default_rng(3)
    Z = layer_norm(rng.standard_normal((5, 64)) * 3 + 1, np.ones(64), np.zeros(64))
    assert np.max(np.abs(Z.mean(axis=1))) < 1e-12
    assert np.max(np.abs(Z.var(axis=1) - 1.0)) < 1e-5


def pin_silu_swiglu(steps=None):
    del steps
    assert silu(np.array(0.0)) == 0.0
    assert abs(silu(np.array(1.0)) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(silu(np.array(-2.0)) - (-2.0 / (1.0 + math.exp(2.0)))) < 1e-15
    rng = np.random.default_rng(5)
    z = rng.standard_normal(3)
    W1, W3, W2 = rng.standard_normal((3, 2)), rng.standard_normal((3, 2)), rng.standard_normal((2, 3))
    want = _bf_ffn(z.tolist(), W1.tolist(), W3.tolist(), W2.tolist())
    assert np.max(np.abs(swiglu_ffn(z, W1, W3, W2) - want)) < 1e-13


def pin_stack_bruteforce(steps=None):
    rng = np.random.default_rng(7)
    for lens, k, d, h in [([5, 0, 3], 3, 4, 6), ([4, 6], 2, 3, 4)]:
        offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        X = rng.standard_normal((offs[-1], d))
        P = rng.standard_normal((k, d))
        layers = [_params(rng, d, h), _params(rng, d, h)]
        got = refine_stack(X, offs, P, layers, steps=steps)
        want = _bf_stack(X, offs, P, layers)
        for b in range(len(lens)):
            if lens[b] == 0:
                continue
            assert np.max(np.abs(got[b] - np.array(want[b]))) < 1e-10, f"user {b}"


def pin_uniform_assignment_mean(steps=None):
    """W_Q = 0 and a zero FFN: A = 1/k, so X-bar_j = LN1(prev_j + mean of the
    user's rows) and the layer output is LN2 of that."""
    rng = np.random.default_rng(11)
    d, k, h = 6, 4, 8
    X = rng.standard_normal((30, d))
    offs = np.array([0, 30], np.int64)
    P = rng.standard_normal((k, d))
    L = _params(rng, d, h, zero_ffn=True, zero_wq=True)
    got = refine_stack(X, offs, P, [L], steps=steps)[0]
    mean = X.mean(axis=0)
    for j in range(k):
        xbar = _bf_ln((P[j] + mean).tolist(), L["gamma1"].tolist(), L["beta1"].tolist())
        want = _bf_ln(xbar, L["gamma2"].tolist(), L["beta2"].tolist())
        assert np.max(np.abs(got[j] - np.array(want))) < 1e-10


def pin_hard_assignment_centroids(steps=None):
    """Huge scale, zero FFN, gamma = 1, beta = 0: X-bar_j is LN1 of P_j plus
    the k-means centroid of the rows whose best prototype is j."""
    rng = np.random.default_rng(13)
    n, k, d = 300, 5, 8
    X = rng.standard_normal((n, d))
    P = rng.standard_normal((k, d))
    L = _params(rng, d, 8, scale=5e3, zero_ffn=True)
    for key in ("gamma1", "gamma2"):
        L[key] = np.ones(d)
    for key in ("beta1", "beta2"):
        L[key] = np.zeros(d)
    logits = X @ (L["W_K"] @ (L["W_Q"].T @ P.T))
    top2 = np.sort(logits, axis=1)[:, -2:]
    keep = (top2[:, 1] - top2[:, 0]) > 0.02
    X, logits = X[keep], logits[keep]
    assign = np.argmax(logits, axis=1)
    offs = np.array([0, len(X)], np.int64)
    got = refine_stack(X, offs, P, [L], steps=steps)[0]
    for j in range(k):
        rows = X[assign == j]
        M = rows.mean(axis=0) if len(rows) else np.zeros(d)
        xbar = _bf_ln((P[j] + M).tolist(), [1.0] * d, [0.0] * d)
        want = _bf_ln(xbar, [1.0] * d, [0.0] * d)
        assert np.max(np.abs(got[j] - np.array(want))) < 1e-8, f"prototype {j}"


def pin_permutations(steps=None):
    rng = np.random.default_rng(17)
    n, k, d, h = 25, 5, 6, 8
    X = rng.standard_normal((n, d))
    P = rng.standard_normal((k, d))
    layers = [_params(rng, d, h), _params(rng, d, h)]
    offs = np.array([0, n], np.int64)
    base = refine_stack(X, offs, P, layers, steps=steps)[0]
    pr = rng.permutation(n)
    assert np.max(np.abs(refine_stack(X[pr], offs, P, layers, steps=steps)[0] - base)) < 1e-10
    pj = rng.permutation(k)
    assert np.max(np.abs(refine_stack(X, offs, P[pj], layers, steps=steps)[0] - base[pj])) < 1e-10


PINS = [pin_layer_norm, pin_silu_swiglu, pin_stack_bruteforce, pin_uniform_assignment_mean,
        pin_hard_assignment_centroids, pin_permutations]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_refine_oracle_satisfies_pin(pin):
    pin()


def _ln_wrong_axis(Z, g, b, eps=LN_EPS):
    Z = np.asarray(Z, np.float64)
    mu = Z.mean(axis=-2, keepdims=True)
    var = ((Z - mu) ** 2).mean(axis=-2, keepdims=True)
    return (Z - mu) / np.sqrt(var + eps) * g + b


def _ln_no_eps(Z, g, b, eps=LN_EPS):
    return layer_norm(Z, g, b, eps=0.0)


def _ffn_gate_swapped(Z, W1, W3, W2):
    return swiglu_ffn(Z, W3, W1, W2)


MUTANTS = {
    "LN over the prototype axis": dict(norm=_ln_wrong_axis),
    "LN without eps": dict(norm=_ln_no_eps),
    "input residual dropped": dict(residual_in=lambda prev, M: M),
    "raw sum in place of the mass-normalised sketch":
        dict(aggregate=lambda Xt, m: np.asarray(Xt, np.float64)),
    "SiLU on the linear branch": dict(ffn=_ffn_gate_swapped),
    "FFN residual dropped": dict(residual_ffn=lambda Xbar, F: F),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_refine_mutant_is_caught(name):
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(steps=MUTANTS[name])
        except (AssertionError, ValueError, FloatingPointError, ZeroDivisionError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name!r} passed every pin"
