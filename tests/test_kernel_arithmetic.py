"""The bf16 path's rounding points, emulated in numpy, against the oracle.

The tolerances the GPU parity tests apply (reading R9: 2e-2 of the user's
largest |X~| and largest m; |sum_j m_j - n_b| <= 2^-8 n_b) are only useful if
a correct implementation of the kernel's arithmetic lands well inside them
and a plausible mistake lands outside.  This test emulates that arithmetic
on the workloads' shapes and value distributions:

  Q' = bf16(P W_Q W_K^T * scale * log2 e)      (fp64 product, one rounding)
  S  = fp32(X Q'^T)                            (bf16 X; exact products, fp32 result)
  e  = exp2(S - max_j S), z = fp32 sum          (section 2.1: the softmax runs
  p  = bf16(e / z)                              over the prototypes)
  X~ = p^T X,  m = sum_i p                      (fp32 accumulation of the same p)

and, for more than 128 prototypes, the slice combination of the clusters
(L_h = m_h + log2 z_h, M = max L_h, Z = sum 2^(L_h - M), factor
2^(m_h - M) / Z).  It checks a margin of at least 4x under each bar, and
that normalising each slice on its own (a plausible cluster mistake) fails.
"""

import math

import numpy as np
import pytest

from oracle import sa_user
from synthetic import generate
from synthetic.workloads import make_inputs, round_to_bf16

LOG2E = 1.0 / math.log(2.0)
TOL = 2e-2
MASS_TOL = 2.0 ** -8


def _bf16(a):
    return round_to_bf16(np.asarray(a, np.float32)).astype(np.float64)


def emulate(Xb, P, W_Q, W_K, scale, slice_len=None, independent_slices=False):
    Qp = _bf16((np.asarray(P, np.float64) @ W_Q @ np.asarray(W_K, np.float64).T) * scale * LOG2E)
    S = (np.asarray(Xb, np.float64) @ Qp.T).astype(np.float32)         # n x k
    k = S.shape[1]
    if slice_len is None or slice_len >= k:
        t = S - S.max(axis=1, keepdims=True)
        e = np.exp2(t.astype(np.float64)).astype(np.float32)
        z = e.sum(axis=1, keepdims=True, dtype=np.float32)
        p = _bf16(e * (np.float32(1.0) / z))
    else:
        C = -(-k // slice_len)
        parts, L, mh = [], [], []
        for h in range(C):
            Sh = S[:, h * slice_len:(h + 1) * slice_len]
            m_h = Sh.max(axis=1, keepdims=True)
            e_h = np.exp2((Sh - m_h).astype(np.float64)).astype(np.float32)
            z_h = e_h.sum(axis=1, keepdims=True, dtype=np.float32)
            parts.append((e_h, z_h))
            mh.append(m_h)
            L.append((m_h + np.log2(z_h)).astype(np.float32))
        M = np.max(np.concatenate(L, axis=1), axis=1, keepdims=True)
        Z = np.zeros_like(M)
        for h in range(C):
            Z += np.exp2((L[h] - M).astype(np.float64)).astype(np.float32)
        ps = []
        for h in range(C):
            e_h, z_h = parts[h]
            f = (np.float32(1.0) / z_h) if independent_slices else \
                (np.exp2((mh[h] - M).astype(np.float64)).astype(np.float32) / Z)
            ps.append(_bf16(e_h * f))
        p = np.concatenate(ps, axis=1)
    Xt = (p.T @ np.asarray(Xb, np.float64)).astype(np.float32).astype(np.float64)
    m = p.sum(axis=0, dtype=np.float32).astype(np.float64)
    return Xt, m


def _errors(Xt, m, Xo, mo, n):
    ex = np.abs(Xt - Xo).max() / np.abs(Xo).max()
    em = np.abs(m - mo).max() / np.abs(mo).max()
    es = abs(m.sum() - n) / n
    return ex, em, es


@pytest.mark.parametrize("workload,rows", [("batch16_n100k_d128_k128_mixture_bf16", 12000),
                                           ("batch32_n10k_d128_k64_bf16", 10000)])
def test_kernel_arithmetic_is_well_inside_the_bars(workload, rows):
    inp = generate(workload)
    Xb = inp["X"][:rows]
    Xt, m = emulate(Xb, inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
    Xo, mo = sa_user(Xb, inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
    ex, em, es = _errors(Xt, m, Xo, mo, rows)
    assert ex < TOL / 4 and em < TOL / 4, (ex, em)
    assert es < MASS_TOL / 4, es


def test_cluster_slices_are_well_inside_the_bars_and_a_slice_mistake_is_not():
    inp = make_inputs([6000], d=128, k=1000, dtype="bf16", seed=71, x_kind="mixture")
    Xb = inp["X"]
    Xo, mo = sa_user(Xb, inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
    Xt, m = emulate(Xb, inp["P"], inp["W_Q"], inp["W_K"], inp["scale"], slice_len=128)
    ex, em, es = _errors(Xt, m, Xo, mo, Xb.shape[0])
    assert ex < TOL / 4 and em < TOL / 4 and es < MASS_TOL / 4, (ex, em, es)
    Xt, m = emulate(Xb, inp["P"], inp["W_Q"], inp["W_K"], inp["scale"], slice_len=128,
                    independent_slices=True)
    ex, em, es = _errors(Xt, m, Xo, mo, Xb.shape[0])
    assert ex > TOL and es > MASS_TOL, (ex, es)
