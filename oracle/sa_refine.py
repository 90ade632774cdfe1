"""CPU oracle for the stacked refinement layers of Sketch Attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library.  Plain numpy, float64.

Source: the reading notes "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模",
section 2.2 "Stacked Refinement 与动作侧融合".  The page lost the layer's
formulas (paper eqs. 10-14); what remains fixes:

* layer l starts from X~^(0) = P^(0) and queries the ORIGINAL history X again
  with the previous layer's sketch (not self-attention over the sketch);
* A^(l) is that layer's assignment (the section 2.1 softmax over prototypes);
* X-bar is the intermediate state "after adding the history aggregation and
  normalising"; LN is layer normalisation; FFN is a feed-forward network;
* the residual keeps the existing representation, the FFN adds capacity
  beyond a linear sum; the final configuration has two layers, width 128 and
  about a thousand prototypes.

Readings where the page is silent:
  F1  the aggregation enters the residual as the mass-normalised sketch
      X~_j / m_j (the weighted mean of the user's rows under prototype j; 0
      where m_j = 0).  The raw sum A X grows with the history length (about
      n / k rows' worth per prototype), so added to X~^(l-1) it would drown
      the residual the page says is kept.
  F2  post-norm:  X-bar = LN(X~^(l-1) + X~_j / m_j),
                  X~^(l) = LN(X-bar + FFN(X-bar)),
      LN over the feature axis (width d) with gain gamma and shift beta,
      biased variance, eps = 1e-5.
  F3  FFN(z) = (SiLU(z W_1) * (z W_3)) W_2, the SwiGLU-gated feed-forward
      network the same section names for action fusion, with hidden width h
      (a parameter; 4 d in the workloads) and no biases (reading R2: the
      page writes no bias anywhere).  SiLU(x) = x / (1 + e^-x).
  F4  every layer has its own W_Q, W_K, LN and FFN parameters (the page does
      not say they are shared; a caller that wants sharing passes the same
      arrays).
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

from .sa_oracle import mass_normalised, sa_batch, sa_batch_user_queries

F64 = np.float64
LN_EPS = 1e-5


def layer_norm(Z: np.ndarray, gamma: np.ndarray, beta: np.ndarray,
               eps: float = LN_EPS) -> np.ndarray:
    """LN over the last axis: (z - mean) / sqrt(var + eps) * gamma + beta,
    var the biased variance (reading F2)."""
    Z = np.asarray(Z, F64)
    mu = Z.mean(axis=-1, keepdims=True)
    var = ((Z - mu) ** 2).mean(axis=-1, keepdims=True)
    return (Z - mu) / np.sqrt(var + eps) * np.asarray(gamma, F64) + np.asarray(beta, F64)


def silu(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, F64)
    return x / (1.0 + np.exp(-x))


def swiglu_ffn(Z: np.ndarray, W1: np.ndarray, W3: np.ndarray, W2: np.ndarray) -> np.ndarray:
    """(SiLU(Z W1) * (Z W3)) W2 over the last axis (reading F3).  W1, W3 are
    d x h, W2 is h x d."""
    Z = np.asarray(Z, F64)
    return (silu(Z @ np.asarray(W1, F64)) * (Z @ np.asarray(W3, F64))) @ np.asarray(W2, F64)


def _residual_in(prev, M):
    return np.asarray(prev, F64) + M


def _residual_ffn(Xbar, F):
    return Xbar + F


DEFAULT_STEPS = dict(norm=layer_norm, ffn=swiglu_ffn, aggregate=mass_normalised,
                     residual_in=_residual_in, residual_ffn=_residual_ffn)


def refine_update(prev: np.ndarray, Xt: np.ndarray, m: np.ndarray,
                  params: Dict[str, np.ndarray], steps=None) -> np.ndarray:
    """The part of a refinement layer after its SA step, for every user:
    X-bar = LN1(prev + X~/m), out = LN2(X-bar + FFN(X-bar)).  prev, Xt are
    (..., k, d), m is (..., k).  Readings F1-F3.  ``steps`` lets tests
    substitute a step (to show that the pins catch a planted mistake)."""
    st = DEFAULT_STEPS if steps is None else {**DEFAULT_STEPS, **steps}
    M = st["aggregate"](Xt, m)
    Xbar = st["norm"](st["residual_in"](prev, M), params["gamma1"], params["beta1"])
    F = st["ffn"](Xbar, params["W1"], params["W3"], params["W2"])
    return st["norm"](st["residual_ffn"](Xbar, F), params["gamma2"], params["beta2"])


def refine_layer(X: np.ndarray, offsets: Sequence[int], prev: Optional[np.ndarray],
                 P: np.ndarray, layer: Dict[str, np.ndarray],
                 users: Optional[Sequence[int]] = None, steps=None) -> np.ndarray:
    """One refinement layer over a ragged batch.  prev is the previous
    layer's sketches (B x k x d); None means the first layer, whose query
    and residual are the shared prototypes P^(0) (X~^(0) = P^(0)).  `layer`
    holds W_Q, W_K, scale and the parameters of refine_update.  Returns
    B x k x d (users not in `users` stay 0)."""
    offsets = np.asarray(offsets, np.int64)
    B = len(offsets) - 1
    k, d = np.shape(P)
    if prev is None:
        Xt, m = sa_batch(X, offsets, P, layer["W_Q"], layer["W_K"], layer["scale"], users=users)
        prev = np.broadcast_to(np.asarray(P, F64), (B, k, d))
    else:
        Xt, m = sa_batch_user_queries(X, offsets, prev, layer["W_Q"], layer["W_K"],
                                      layer["scale"], users=users)
    out = np.zeros((B, k, d), F64)
    for b in (range(B) if users is None else users):
        out[b] = refine_update(prev[b], Xt[b], m[b], layer, steps=steps)
    return out


def refine_stack(X: np.ndarray, offsets: Sequence[int], P: np.ndarray,
                 layers: Sequence[Dict[str, np.ndarray]],
                 users: Optional[Sequence[int]] = None, steps=None) -> np.ndarray:
    """N_sa stacked refinement layers (section 2.2): layer 1 from P^(0),
    each later layer queried by the previous layer's sketches; every layer
    reads the original X.  Returns X~^(N_sa), B x k x d."""
    prev = None
    for layer in layers:
        prev = refine_layer(X, offsets, prev, P, layer, users=users, steps=steps)
    return prev
