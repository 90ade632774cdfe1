"""CPU oracle for the gradients of one SA layer (test infrastructure only).

Same rules as ``sa_oracle``: plain numpy in float64, no code shared with the
CUDA library; only ``tests/`` may import it.

Source: the reading notes "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模",
section 2.2: the compression module sits in the training path and is trained
by gradient descent on the final ranking objective ("end to end").  The page
gives no backward formulas; they follow from the forward of section 2.1 by
the chain rule, step by step in the forward's order (reversed):

    K = X W_K,  Q = P W_Q,  S = Q K^T scale,
    A = softmax of S over the prototype axis (every column sums to 1),
    X~ = A X,  m = A 1.

Given the upstream gradients G = dL/dX~ (k x d) and g = dL/dm (k):

    dA  = G X^T + g 1^T                          (k x n)
    dS  = A * (dA - 1 c^T),  c_i = sum_j A_ji dA_ji   (softmax over axis 0)
    dQ  = scale dS K,        dK = scale dS^T Q
    dP  = dQ W_Q^T,          dW_Q = P^T dQ
    dX  = A^T G + dK W_K^T,  dW_K = X^T dK

Readings (the page prints no backward pass):
  B1  the loss may depend on both outputs, X~ and m (m is returned beside X~,
      reading R4), so both upstream gradients are inputs; g = 0 gives the
      gradient of a loss on X~ alone.
  B2  scale is a constant (reading R2): it gets no gradient.
  B3  with per-user queries (reading R12) the query matrix Q_b takes P's
      place, so dQ_b is this function's dP for that user.
  B4  gradients of a batch are per user for X and P-like inputs, and summed
      over users for the shared W_Q, W_K (and P, when P is shared).

Pinned in tests/test_oracle_backward.py against central finite differences of
the forward oracle, a closed form for k = 1 and the zero-gradient cases.
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

F64 = np.float64


def sa_user_backward(Xb: np.ndarray, P: np.ndarray, W_Q: np.ndarray, W_K: np.ndarray,
                     scale: float, G: np.ndarray, g: Optional[np.ndarray] = None
                     ) -> Dict[str, np.ndarray]:
    """Gradients of one user's SA layer.

    Xb (n x d), P (k x d), W_Q, W_K (d x d); G = dL/dX~ (k x d), g = dL/dm (k,)
    or None (zero).  Returns dX (n x d), dP (k x d), dW_Q, dW_K (d x d), all
    float64.  An empty history gives zero gradients (reading R5).
    """
    Xb = np.asarray(Xb, F64)
    P = np.asarray(P, F64)
    W_Q = np.asarray(W_Q, F64)
    W_K = np.asarray(W_K, F64)
    G = np.asarray(G, F64)
    k, d = P.shape
    g = np.zeros(k, F64) if g is None else np.asarray(g, F64)
    n = Xb.shape[0]
    if n == 0:
        return dict(dX=np.zeros((0, d), F64), dP=np.zeros((k, d), F64),
                    dW_Q=np.zeros((d, d), F64), dW_K=np.zeros((d, d), F64))
    # forward, kept for the backward
    K = Xb @ W_K
    Q = P @ W_Q
    S = (Q @ K.T) * F64(scale)
    E = np.exp(S - S.max(axis=0, keepdims=True))
    A = E / E.sum(axis=0, keepdims=True)
    # backward, in reverse order
    dA = G @ Xb.T + g[:, None]
    c = (A * dA).sum(axis=0, keepdims=True)
    dS = A * (dA - c)
    dQ = F64(scale) * (dS @ K)
    dK = F64(scale) * (dS.T @ Q)
    return dict(dX=A.T @ G + dK @ W_K.T, dP=dQ @ W_Q.T, dW_Q=P.T @ dQ, dW_K=Xb.T @ dK)


def sa_batch_backward(X: np.ndarray, offsets: Sequence[int], P: np.ndarray, W_Q: np.ndarray,
                      W_K: np.ndarray, scale: float, G: np.ndarray,
                      g: Optional[np.ndarray] = None, queries: Optional[np.ndarray] = None
                      ) -> Dict[str, np.ndarray]:
    """Gradients of a ragged batch (user b owns rows offsets[b]..offsets[b+1]).

    G (B x k x d), g (B x k) or None.  With ``queries`` (B x k x d) user b is
    queried by queries[b] (reading B3) and the result holds dQueries (B x k x
    d) in place of dP; otherwise dP (k x d) is summed over users (B4).
    Returns dX (N x d), dP or dQueries, dW_Q and dW_K (summed over users).
    """
    offsets = np.asarray(offsets, np.int64)
    X = np.asarray(X, F64)
    B = len(offsets) - 1
    k, d = np.shape(P) if queries is None else np.shape(queries)[1:]
    dX = np.zeros_like(X)
    dW_Q = np.zeros((d, d), F64)
    dW_K = np.zeros((d, d), F64)
    dP = np.zeros((k, d), F64)
    dQs = np.zeros((B, k, d), F64)
    for b in range(B):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        Pb = P if queries is None else queries[b]
        r = sa_user_backward(X[lo:hi], Pb, W_Q, W_K, scale, G[b], None if g is None else g[b])
        dX[lo:hi] = r["dX"]
        dW_Q += r["dW_Q"]
        dW_K += r["dW_K"]
        if queries is None:
            dP += r["dP"]
        else:
            dQs[b] = r["dP"]
    out = dict(dX=dX, dW_Q=dW_Q, dW_K=dW_K)
    if queries is None:
        out["dP"] = dP
    else:
        out["dQueries"] = dQs
    return out
