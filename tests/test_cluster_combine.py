"""Reading R13 on the CPU: the softmax over k prototypes computed in slices
of 128 (what a cluster of CTAs does, each holding one slice) is the softmax
over the whole prototype axis (section 2.1 of the SequenceO1 reading notes:
the normaliser sums over every prototype).

Each slice h reports its maximum m_h and sum z_h = sum_j 2^(t_j - m_h) as one
value L_h = m_h + log2 z_h; with M = max_h L_h and Z = sum_h 2^(L_h - M), the
weights of slice h are 2^(t_j - m_h) * 2^(m_h - M) / Z.  Logits t are in
base-2 units (t = s log2 e), so the result must equal the oracle's
exp-based softmax of s.  This checks the identity, in fp64, not a kernel."""

import numpy as np
import pytest

from oracle import prototype_softmax

LOG2E = 1.0 / np.log(2.0)


def sliced_softmax(T, slice_len=128, k_valid=None):
    """Columns are behaviours, rows prototypes (k x n), base-2 logits."""
    k, n = T.shape
    k_valid = k if k_valid is None else k_valid
    T = T.copy()
    T[k_valid:] = -np.inf                      # padded prototypes
    C = -(-k // slice_len)
    m = np.empty((C, n))
    L = np.empty((C, n))
    E = np.empty_like(T)
    for h in range(C):
        sl = slice(h * slice_len, min(k, (h + 1) * slice_len))
        m[h] = T[sl].max(axis=0)
        with np.errstate(invalid="ignore"):
            E[sl] = np.where(np.isfinite(T[sl]), np.exp2(T[sl] - m[h]), 0.0)
        z = E[sl].sum(axis=0)
        with np.errstate(divide="ignore"):
            L[h] = m[h] + np.log2(z)            # -inf for a slice of padding only
    M = L.max(axis=0)
    Z = np.zeros(n)
    for h in range(C):                          # rank order
        Z += np.exp2(L[h] - M)
    A = np.empty_like(T)
    for h in range(C):
        sl = slice(h * slice_len, min(k, (h + 1) * slice_len))
        with np.errstate(invalid="ignore"):
            f = np.where(np.isfinite(m[h]), np.exp2(m[h] - M), 0.0) / Z
        A[sl] = E[sl] * f
    return A[:k_valid]


@pytest.mark.parametrize("k,k_valid", [(256, 256), (1024, 1000), (384, 300), (512, 257)])
def test_sliced_softmax_equals_softmax_over_all_prototypes(k, k_valid):
    rng = np.random.default_rng(k + k_valid)
    S = rng.standard_normal((k_valid, 333)) * 4.0
    S[:, 7] += 900.0                            # large logits stay finite
    S[3, 11] = 60.0                             # one prototype dominates a row
    T = np.full((k, S.shape[1]), -np.inf)
    T[:k_valid] = S * LOG2E
    A = sliced_softmax(T, k_valid=k_valid)
    np.testing.assert_allclose(A, prototype_softmax(S), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(A.sum(axis=0), 1.0, rtol=1e-12)


def test_a_wrong_combination_is_caught():
    # Normalising each slice on its own (no cross-slice total) is not the
    # softmax over all prototypes.
    rng = np.random.default_rng(5)
    S = rng.standard_normal((256, 50))
    A_bad = np.concatenate([prototype_softmax(S[:128]), prototype_softmax(S[128:])])
    assert not np.allclose(A_bad, prototype_softmax(S))
    T = S * LOG2E
    assert np.allclose(sliced_softmax(T), prototype_softmax(S))
