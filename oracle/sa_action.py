"""CPU oracle for action-side fusion, the producer of the history matrix X.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library.  Plain numpy, float64.

Source: the reading notes "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模",
section 2.2 "Stacked Refinement 与动作侧融合".  The page lost the formula
itself; its symbol list fixes what it computes: e_i is the item embedding of
the i-th behaviour, a_i the embedding of its action type (finish, swipe,
like, follow ... give the same video different meanings), the two are
concatenated, a SwiGLU-gated feed-forward network maps the concatenation
back to the item width, and the result is added to e_i as a residual:

    x_i = e_i + FFN([e_i ; a_i]),    FFN(z) = (SiLU(z W_1) * (z W_3)) W_2.

Only x_i enters the history matrix X that Sketch Attention compresses, so
the action meaning is attached to each video before aggregation.

Readings where the page is silent:
  A1  a_i is the row of an action-type embedding table (n_types x d_a) that
      the behaviour's type id selects; one type per behaviour.
  A2  the FFN is the SwiGLU form above (reading F3 of the refinement layers)
      with no biases (reading R2), hidden width h a parameter; W_1, W_3 are
      (d + d_a) x h with the e-rows first (the concatenation order [e ; a]),
      W_2 is h x d.
  A3  e_i arrives as a row of the producer's input (the lookup of the item
      table is upstream of this step); any production feature transforms
      beyond this abstract form are out of scope (the page says the
      production version may have more).
"""

from __future__ import annotations

import numpy as np

from .sa_refine import silu

F64 = np.float64


def fusion_input(E: np.ndarray, types: np.ndarray, table: np.ndarray) -> np.ndarray:
    """z_i = [e_i ; a_i] with a_i = table[types[i]] (readings A1, A2)."""
    E = np.asarray(E, F64)
    A = np.asarray(table, F64)[np.asarray(types, np.int64)]
    return np.concatenate([E, A], axis=-1)


def fusion_hidden(Z: np.ndarray, W1: np.ndarray, W3: np.ndarray):
    """The FFN's gate input u = z W_1, value v = z W_3 and gated hidden
    g = SiLU(u) * v."""
    U = np.asarray(Z, F64) @ np.asarray(W1, F64)
    V = np.asarray(Z, F64) @ np.asarray(W3, F64)
    return U, V, silu(U) * V


def action_fuse(E: np.ndarray, types: np.ndarray, table: np.ndarray, W1: np.ndarray,
                W3: np.ndarray, W2: np.ndarray) -> np.ndarray:
    """x_i = e_i + (SiLU(z_i W_1) * (z_i W_3)) W_2 with z_i = [e_i ; a_i]
    for every row i of E (n x d); returns X (n x d), float64."""
    _, _, G = fusion_hidden(fusion_input(E, types, table), W1, W3)
    return np.asarray(E, F64) + G @ np.asarray(W2, F64)
