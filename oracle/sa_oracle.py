"""CPU oracle for the Sketch Attention (SA) compression step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The CUDA library never calls it, and it imports nothing from the
CUDA package: the two share no code.  It is plain, slow and fp64 on purpose.

Source: the reading notes "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模"
(on "SequenceO1: End-to-End Ultra-Long (100K) Sequence Modeling in
Recommendation with Low-Rank Caching"), section 2.1 "Sketch Attention".
The page lost its display formulas (paper eqs. 6-9) in extraction; what
remains fixes the computation:

* X in R^{n x d} is the user history (rows are behaviours), P^(0) in
  R^{k x d} the shared learnable prototypes, W_Q, W_K in R^{d x d} the
  projections; S in R^{k x n} is the prototype-behaviour affinity, j indexes
  prototypes and i behaviours.
* The normaliser sums over the prototype index, so every behaviour spreads
  unit weight over the k prototypes (section 2.1, symbol explanation).
* The sketch aggregates X itself; no value projection is applied
  (section 2.1, symbol explanation).
* The sketch is a weighted aggregation, not a selection; prototypes are not
  forced to receive equal mass (section 2.1, closing paragraph).

Readings where the page is silent:
  R1  S = (P W_Q)(X W_K)^T * scale, i.e. S_ji = scale * (p_j W_Q).(x_i W_K).
  R2  scale is an input (1/sqrt(d) in every workload); no learnable
      temperature, no projection bias.
  R3  the softmax is made stable by subtracting, per behaviour, the largest
      logit over prototypes (section 2.4: FlashSA keeps "stable softmax
      statistics"); the result is the same function.
  R4  the per-prototype mass m_j = sum_i A_ji is returned next to the sketch
      so that a mass-normalised sketch X~_j / m_j can be derived.
  R5  a user with no rows has X~ = 0 and m = 0; rows outside a user's range
      contribute nothing to it (section 3.1: padding must not be assigned
      mass).
  R12 (section 2.2) a refinement layer's SA step queries user b's rows with
      that user's previous sketch in place of P^(0) (sa_batch_user_queries).

Every function works in float64; float32 / bf16 inputs are upcast exactly.
"""

from __future__ import annotations

from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# The steps of one SA layer, in the order of section 2.1
# ---------------------------------------------------------------------------

def project_keys(Xb: np.ndarray, W_K: np.ndarray) -> np.ndarray:
    """K = X W_K  (n x d).  The oracle materialises the key projection that
    the fast path avoids by reassociation (section 1 notes the same
    rearrangement for single-query cross-attention)."""
    return np.asarray(Xb, F64) @ np.asarray(W_K, F64)


def project_prototypes(P: np.ndarray, W_Q: np.ndarray) -> np.ndarray:
    """Q = P^(0) W_Q  (k x d)."""
    return np.asarray(P, F64) @ np.asarray(W_Q, F64)


def affinity(Q: np.ndarray, K: np.ndarray, scale: float) -> np.ndarray:
    """S = Q K^T * scale  (k x n): row j is prototype j, column i behaviour i
    (reading R1)."""
    return (Q @ K.T) * F64(scale)


def prototype_softmax(S: np.ndarray) -> np.ndarray:
    """A_ji = exp(S_ji - c_i) / sum_j' exp(S_j'i - c_i),  c_i = max_j S_ji.

    The denominator runs over the prototype index j (axis 0), so every column
    of A sums to one (section 2.1, symbol explanation; reading R3)."""
    c = S.max(axis=0, keepdims=True)
    E = np.exp(S - c)
    return E / E.sum(axis=0, keepdims=True)


def aggregate(A: np.ndarray, Xb: np.ndarray) -> np.ndarray:
    """X~ = A X  (k x d), no value projection (section 2.1)."""
    return A @ np.asarray(Xb, F64)


def prototype_mass(A: np.ndarray) -> np.ndarray:
    """m_j = sum_i A_ji  (reading R4)."""
    return A.sum(axis=1)


DEFAULT_STEPS: Dict[str, Callable] = dict(
    project_keys=project_keys,
    project_prototypes=project_prototypes,
    affinity=affinity,
    prototype_softmax=prototype_softmax,
    aggregate=aggregate,
    prototype_mass=prototype_mass,
)


def sa_user(Xb: np.ndarray, P: np.ndarray, W_Q: np.ndarray, W_K: np.ndarray,
            scale: float, steps: Optional[Dict[str, Callable]] = None,
            return_assignment: bool = False):
    """One SA layer over one user's history Xb (n x d).

    Returns (X~ (k x d), m (k,)) in float64, plus A (k x n) if asked.
    ``steps`` lets tests substitute a step (used to show that the pins catch
    a planted mistake); it defaults to the functions above.
    """
    st = DEFAULT_STEPS if steps is None else {**DEFAULT_STEPS, **steps}
    Xb = np.asarray(Xb, F64)
    k, d = np.shape(P)
    if Xb.shape[0] == 0:  # reading R5
        z = (np.zeros((k, d), F64), np.zeros(k, F64))
        return z + (np.zeros((k, 0), F64),) if return_assignment else z
    K = st["project_keys"](Xb, W_K)
    Q = st["project_prototypes"](P, W_Q)
    S = st["affinity"](Q, K, scale)
    A = st["prototype_softmax"](S)
    Xt = st["aggregate"](A, Xb)
    m = st["prototype_mass"](A)
    return (Xt, m, A) if return_assignment else (Xt, m)


def sa_batch(X: np.ndarray, offsets: Sequence[int], P: np.ndarray,
             W_Q: np.ndarray, W_K: np.ndarray, scale: float,
             users: Optional[Sequence[int]] = None,
             steps: Optional[Dict[str, Callable]] = None
             ) -> Tuple[np.ndarray, np.ndarray]:
    """SA over a ragged batch: user b owns rows [offsets[b], offsets[b+1]).

    Returns X~ (B x k x d) and m (B x k) in float64.  If ``users`` is given,
    only those users are computed (the others stay zero), which is how the
    full-size tests sample outputs.  Only a user's own rows enter its sketch
    (reading R5).
    """
    offsets = np.asarray(offsets, np.int64)
    B = len(offsets) - 1
    k, d = np.shape(P)
    Xt = np.zeros((B, k, d), F64)
    m = np.zeros((B, k), F64)
    for b in (range(B) if users is None else users):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        Xt[b], m[b] = sa_user(X[lo:hi], P, W_Q, W_K, scale, steps=steps)
    return Xt, m


def sa_batch_user_queries(X: np.ndarray, offsets: Sequence[int], queries: np.ndarray,
                          W_Q: np.ndarray, W_K: np.ndarray, scale: float,
                          users: Optional[Sequence[int]] = None
                          ) -> Tuple[np.ndarray, np.ndarray]:
    """SA with a query matrix per user: user b's rows are queried by
    ``queries[b]`` (k x d) in place of the shared P^(0).

    Section 2.2 "Stacked Refinement" of the same notes: refinement layer l
    starts from X~^(0) = P^(0) and each layer still reads the original X,
    queried by the previous layer's sketch.  Reading R12: layer l's SA step
    for user b is the section 2.1 computation with X~_b^(l-1) in place of
    P^(0), with the same W_Q, W_K and scale arguments (whether the
    projections differ per layer is left to the caller, who passes them).
    Returns X~ (B x k x d) and m (B x k) in float64.
    """
    offsets = np.asarray(offsets, np.int64)
    queries = np.asarray(queries)
    B = len(offsets) - 1
    _, k, d = queries.shape
    Xt = np.zeros((B, k, d), F64)
    m = np.zeros((B, k), F64)
    for b in (range(B) if users is None else users):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        Xt[b], m[b] = sa_user(X[lo:hi], queries[b], W_Q, W_K, scale)
    return Xt, m


def mass_normalised(Xt: np.ndarray, m: np.ndarray) -> np.ndarray:
    """X~_j / m_j, defined as 0 where m_j == 0 (reading R4)."""
    m = np.asarray(m, F64)
    safe = np.where(m == 0, 1.0, m)
    return np.where((m == 0)[..., None], 0.0, np.asarray(Xt, F64) / safe[..., None])
