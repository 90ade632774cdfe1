"""The refinement update's rounding points, emulated in numpy, against the
oracle -- the basis of the GPU tolerance for sa_refine_update.

The kernel keeps the norms in fp32 and runs the SwiGLU network on the tensor
cores: z (after LN1) is rounded to bf16 as the MMAs' A operand, the weights
are bf16 copies, H = z W1 and G = z W3 accumulate in fp32, U = SiLU(H) * G
is rounded to bf16 for the second MMA, Y = U W2 accumulates in fp32, and
out = LN2(z + Y) uses the fp32 z.  The GPU tests compare with the oracle per
user with the bar the SA sketches use for bf16 (max |err| <= 2e-2 * max
|oracle|).  This test checks that a faithful emulation of that arithmetic
lands at least 4x inside the bar on the workloads' scales, and that a
plausible mistake (the gate on the wrong branch) lands outside it.
"""

import math

import numpy as np
import pytest

from oracle import refine_update
from synthetic.workloads import round_to_bf16

TOL = 2e-2


def _bf16(a):
    return round_to_bf16(np.asarray(a, np.float32)).astype(np.float32)


def _ln32(Z, g, b):
    Z = Z.astype(np.float32)
    mu = Z.mean(axis=-1, keepdims=True, dtype=np.float32)
    var = ((Z - mu) ** 2).mean(axis=-1, keepdims=True, dtype=np.float32)
    return ((Z - mu) / np.sqrt(var + np.float32(1e-5)) * g.astype(np.float32) +
            b.astype(np.float32)).astype(np.float32)


def emulate(prev, Xt, m, p, swap_gate=False):
    inv = np.where(m > 0, 1.0 / np.where(m > 0, m, 1.0), 0.0).astype(np.float32)
    z = _ln32(prev.astype(np.float32) + Xt.astype(np.float32) * inv[..., None], p["gamma1"],
              p["beta1"])
    zb = _bf16(z).astype(np.float64)
    W1, W3 = _bf16(p["W1"]).astype(np.float64), _bf16(p["W3"]).astype(np.float64)
    if swap_gate:
        W1, W3 = W3, W1
    H = (zb @ W1).astype(np.float32)
    G = (zb @ W3).astype(np.float32)
    U = _bf16(H / (1.0 + np.exp(-H.astype(np.float64))).astype(np.float32) * G)
    Y = (U.astype(np.float64) @ _bf16(p["W2"]).astype(np.float64)).astype(np.float32)
    return _ln32(z + Y, p["gamma2"], p["beta2"])


def _params(rng, d, h):
    return dict(gamma1=1.0 + 0.1 * rng.standard_normal(d), beta1=0.1 * rng.standard_normal(d),
                gamma2=1.0 + 0.1 * rng.standard_normal(d), beta2=0.1 * rng.standard_normal(d),
                W1=rng.standard_normal((d, h)) / math.sqrt(d),
                W3=rng.standard_normal((d, h)) / math.sqrt(d),
                W2=rng.standard_normal((h, d)) / math.sqrt(h))


def _case(seed, B, k, d, h, mass_scale):
    rng = np.random.default_rng(seed)
    prev = rng.standard_normal((B, k, d)).astype(np.float32)
    m = (rng.uniform(0.0, 2.0, (B, k)) * mass_scale).astype(np.float32)
    m[:, :3] = 0.0  # empty prototypes
    # a sketch whose mass-normalised rows are weighted means of N(0,1) rows
    Xt = (rng.standard_normal((B, k, d)) * 0.3 * m[..., None]).astype(np.float32)
    return prev, Xt, m, _params(rng, d, h)


@pytest.mark.parametrize("d,h,mass_scale", [(128, 512, 1e3), (64, 256, 10.0), (128, 128, 1.0)])
def test_refine_arithmetic_is_well_inside_the_bar(d, h, mass_scale):
    prev, Xt, m, p = _case(3, 4, 64, d, h, mass_scale)
    got = emulate(prev, Xt, m, p)
    want = refine_update(prev, Xt, m, p)
    for b in range(prev.shape[0]):
        err = np.abs(got[b] - want[b]).max() / np.abs(want[b]).max()
        assert err < TOL / 4, (b, err)
    bad = emulate(prev, Xt, m, p, swap_gate=True)
    worst = max(np.abs(bad[b] - want[b]).max() / np.abs(want[b]).max() for b in range(4))
    assert worst > TOL, worst
