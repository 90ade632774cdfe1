"""Pure-Python brute force of one SA layer, for tiny inputs only.

TEST INFRASTRUCTURE (same import rule as ``oracle.sa_oracle``).

Written index by index from the definition in section 2.1 "Sketch Attention"
of the SequenceO1 reading notes ("SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模"),
with plain Python floats and loops and no numpy.  It deliberately uses the
textbook softmax (no max subtraction), so it is an independent derivation of
the same numbers rather than a second copy of ``sa_oracle``; keep its inputs
small and their logits moderate.
"""

from __future__ import annotations

import math
from typing import List, Sequence, Tuple


def sa_user_bruteforce(X: Sequence[Sequence[float]], P: Sequence[Sequence[float]],
                       W_Q: Sequence[Sequence[float]], W_K: Sequence[Sequence[float]],
                       scale: float) -> Tuple[List[List[float]], List[float]]:
    n = len(X)
    k = len(P)
    d = len(P[0]) if k else 0
    # key of behaviour i: K_i,e = sum_f X_i,f W_K[f][e]
    K = [[sum(float(X[i][f]) * float(W_K[f][e]) for f in range(d)) for e in range(d)]
         for i in range(n)]
    # query of prototype j: Q_j,e = sum_f P_j,f W_Q[f][e]
    Q = [[sum(float(P[j][f]) * float(W_Q[f][e]) for f in range(d)) for e in range(d)]
         for j in range(k)]
    # affinity S_j,i = scale * sum_e Q_j,e K_i,e
    S = [[scale * sum(Q[j][e] * K[i][e] for e in range(d)) for i in range(n)]
         for j in range(k)]
    # weights: for each behaviour i, normalise over prototypes j
    A = [[0.0] * n for _ in range(k)]
    for i in range(n):
        z = sum(math.exp(S[j][i]) for j in range(k))
        for j in range(k):
            A[j][i] = math.exp(S[j][i]) / z
    # sketch X~_j,e = sum_i A_j,i X_i,e   and mass m_j = sum_i A_j,i
    Xt = [[sum(A[j][i] * float(X[i][e]) for i in range(n)) for e in range(d)]
          for j in range(k)]
    m = [sum(A[j][i] for i in range(n)) for j in range(k)]
    return Xt, m
