"""Seeded generators for the SA workloads (inputs only, no SA arithmetic).

Each workload is a ragged batch of user histories.  Values follow the recipe
below; every draw comes from ``numpy.random.default_rng(seed)`` in a fixed
order (lengths, X, P, W_Q, W_K), so a (workload, seed) pair names one exact
input everywhere.

bf16 workloads are drawn in float32 and then rounded to the nearest bf16
value (round to nearest, ties to even).  The arrays handed out stay float32
(each value exactly representable in bf16); ``bf16_bits`` gives the 16-bit
patterns that the CUDA path consumes.  The oracle upcasts the same float32
values to float64 exactly, so both sides read identical numbers.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named synthetic workload.

    lengths: "uniform" (every user has n rows) or "loguniform" (n_b drawn as
    floor(exp(U(ln lo, ln hi))) per user, no padding).
    x_kind: "normal" (X ~ N(0, 1)) or "mixture" (a Gaussian mixture with
    ``mix_components`` means ~ N(0, I), per-component sd ``mix_sd``, and a
    component drawn i.i.d. uniformly per row).
    """

    name: str
    batch: int
    d: int
    k: int
    dtype: str  # "bf16" or "fp32"
    seed: int
    lengths: str = "uniform"
    n: int = 0
    lo: int = 0
    hi: int = 0
    x_kind: str = "normal"
    mix_components: int = 0
    mix_sd: float = 0.0


# The workloads.  Their shapes are the ones the method is quoted on:
# single users of ~1K rows for the exact fp32 check, batches of 10K- and
# 100K-row histories at width 128 (the final SA width of section 3.2), a
# ragged batch spanning the whole 1K-100K range, a wide d=256/k=256 case
# where the tensor cores rather than HBM bound the step, and the 100K batch
# with about a thousand prototypes.
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("single_n1024_d64_k16_fp32", batch=1, n=1024, d=64, k=16,
                 dtype="fp32", seed=1000),
        Workload("batch32_n10k_d128_k64_bf16", batch=32, n=10_000, d=128, k=64,
                 dtype="bf16", seed=1001),
        Workload("batch16_n100k_d128_k128_mixture_bf16", batch=16, n=100_000,
                 d=128, k=128, dtype="bf16", seed=1002, x_kind="mixture",
                 mix_components=512, mix_sd=0.3),
        Workload("ragged256_loguniform_1k_100k_d128_k64_bf16", batch=256, d=128,
                 k=64, dtype="bf16", seed=1003, lengths="loguniform",
                 lo=1_000, hi=100_000),
        Workload("batch8_n100k_d256_k256_bf16", batch=8, n=100_000, d=256,
                 k=256, dtype="bf16", seed=1004),
        # The 16 x 100K mixture batch at the prototype count of the final
        # refinement layers (about a thousand; section 2.2).
        Workload("batch16_n100k_d128_k1000_mixture_bf16", batch=16, n=100_000,
                 d=128, k=1000, dtype="bf16", seed=1005, x_kind="mixture",
                 mix_components=512, mix_sd=0.3),
    ]
}


# ---------------------------------------------------------------------------
# bf16 helpers (input rounding only)
# ---------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, nearest-even; return the uint16 patterns.

    NaN maps to the quiet NaN 0x7FC0 (sign kept); +-inf stays +-inf.  For
    every non-NaN pattern u <= 0xFF800000 the sum below stays under 2**32,
    so 32-bit arithmetic suffices.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).copy()
    nan = np.isnan(x)
    lsb = (u >> 16) & np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    del lsb
    u >>= 16
    r = u.astype(np.uint16)
    if nan.any():
        sign = (x.view(np.uint32)[nan] >> 16).astype(np.uint16) & np.uint16(0x8000)
        r[nan] = sign | np.uint16(0x7FC0)
    return r.reshape(x.shape)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    """Expand uint16 bf16 patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).reshape(b.shape)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 value, returned as float32."""
    return bf16_from_bits(bf16_bits(x))


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------

def ragged_lengths(rng: np.random.Generator, batch: int, lo: int, hi: int) -> np.ndarray:
    """n_b = floor(exp(U(ln lo, ln hi))) for each user (log-uniform lengths)."""
    u = rng.uniform(math.log(lo), math.log(hi), size=batch)
    return np.floor(np.exp(u)).astype(np.int64)


def _draw_x(rng: np.random.Generator, rows: int, d: int, x_kind: str,
            mix_components: int, mix_sd: float) -> np.ndarray:
    if x_kind == "normal":
        return rng.standard_normal((rows, d), dtype=np.float32)
    if x_kind == "mixture":
        means = rng.standard_normal((mix_components, d), dtype=np.float32)
        comp = rng.integers(0, mix_components, size=rows)
        x = rng.standard_normal((rows, d), dtype=np.float32)
        x *= np.float32(mix_sd)
        x += means[comp]
        return x
    raise ValueError(f"unknown x_kind {x_kind!r}")


def make_inputs(lengths: Sequence[int], d: int, k: int, dtype: str, seed: int,
                x_kind: str = "normal", mix_components: int = 512,
                mix_sd: float = 0.3, scale: Optional[float] = None) -> dict:
    """Draw one ragged batch with the given per-user lengths.

    Returns a dict with X (N, d) float32, offsets (B+1,) int64, P (k, d),
    W_Q (d, d), W_K (d, d) float32, scale (float, default 1/sqrt(d)), dtype.
    For dtype "bf16" every array value is bf16-representable.
    """
    rng = np.random.default_rng(seed)
    return _finish(rng, np.asarray(lengths, dtype=np.int64), d, k, dtype,
                   x_kind, mix_components, mix_sd, scale)


def _finish(rng, lengths, d, k, dtype, x_kind, mix_components, mix_sd, scale):
    if np.any(lengths < 0):
        raise ValueError("negative length")
    offsets = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=offsets[1:])
    n_total = int(offsets[-1])
    X = _draw_x(rng, n_total, d, x_kind, mix_components, mix_sd)
    P = rng.standard_normal((k, d), dtype=np.float32)
    w_sd = np.float32(1.0 / math.sqrt(d))
    W_Q = rng.standard_normal((d, d), dtype=np.float32) * w_sd
    W_K = rng.standard_normal((d, d), dtype=np.float32) * w_sd
    if dtype == "bf16":
        X, P, W_Q, W_K = (round_to_bf16(a) for a in (X, P, W_Q, W_K))
    elif dtype != "fp32":
        raise ValueError(f"unknown dtype {dtype!r}")
    return dict(X=X, offsets=offsets, P=P, W_Q=W_Q, W_K=W_K,
                scale=float(1.0 / math.sqrt(d)) if scale is None else float(scale),
                dtype=dtype, d=d, k=k)


def _draw_lengths(rng: np.random.Generator, w: "Workload") -> np.ndarray:
    if w.lengths == "uniform":
        return np.full(w.batch, w.n, dtype=np.int64)
    if w.lengths == "loguniform":
        return ragged_lengths(rng, w.batch, w.lo, w.hi)
    raise ValueError(w.lengths)


def workload_lengths(name: str, seed: Optional[int] = None) -> np.ndarray:
    """The per-user lengths that ``generate(name, seed)`` draws (its first
    draws), without drawing the rest of the batch."""
    w = WORKLOADS[name]
    return _draw_lengths(np.random.default_rng(w.seed if seed is None else seed), w)


def generate(name: str, seed: Optional[int] = None) -> dict:
    """Draw the named workload (see ``WORKLOADS``) with its own seed."""
    w = WORKLOADS[name]
    rng = np.random.default_rng(w.seed if seed is None else seed)
    lengths = _draw_lengths(rng, w)
    out = _finish(rng, lengths, w.d, w.k, w.dtype, w.x_kind, w.mix_components,
                  w.mix_sd, None)
    out["workload"] = w.name
    return out


def user_queries(batch: int, k: int, d: int, seed: int) -> np.ndarray:
    """Per-user query matrices Q_b (batch, k, d) float32 ~ N(0, 1), the same
    distribution as the shared prototypes P, from their own generator (so a
    workload's other arrays do not change).  They stand in for the previous
    layer's sketch that a refinement layer queries with; they are fp32 (the
    sketch's own type) and not rounded to bf16."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((batch, k, d), dtype=np.float32)


def upstream_gradients(batch: int, k: int, d: int, seed: int):
    """Seeded upstream gradients for an SA layer's backward: G = dL/dX~
    (batch, k, d) and g = dL/dm (batch, k), float64 ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((batch, k, d)), rng.standard_normal((batch, k))


def refine_params(d: int, h: int, seed: int, dtype: str = "bf16") -> dict:
    """Seeded parameters of one refinement layer: W_Q, W_K (d, d) ~ N(0, 1/d)
    (rounded to bf16 for dtype "bf16", like every SA input), and the LN and
    FFN parameters in float32: gamma ~ 1 + 0.1 N(0, 1), beta ~ 0.1 N(0, 1),
    W1, W3 (d, h) ~ N(0, 1/d), W2 (h, d) ~ N(0, 1/h)."""
    rng = np.random.default_rng(seed)
    w_sd = np.float32(1.0 / math.sqrt(d))
    W_Q = rng.standard_normal((d, d), dtype=np.float32) * w_sd
    W_K = rng.standard_normal((d, d), dtype=np.float32) * w_sd
    if dtype == "bf16":
        W_Q, W_K = round_to_bf16(W_Q), round_to_bf16(W_K)
    out = dict(W_Q=W_Q, W_K=W_K, scale=float(1.0 / math.sqrt(d)))
    for g, b in (("gamma1", "beta1"), ("gamma2", "beta2")):
        out[g] = (1.0 + 0.1 * rng.standard_normal(d)).astype(np.float32)
        out[b] = (0.1 * rng.standard_normal(d)).astype(np.float32)
    out["W1"] = (rng.standard_normal((d, h)) / math.sqrt(d)).astype(np.float32)
    out["W3"] = (rng.standard_normal((d, h)) / math.sqrt(d)).astype(np.float32)
    out["W2"] = (rng.standard_normal((h, d)) / math.sqrt(h)).astype(np.float32)
    return out


def action_params(d: int, d_a: int, h: int, n_types: int, seed: int) -> dict:
    """Seeded parameters of the action-fusion producer (x = e + SwiGLU-FFN of
    [e ; a]): the action table (n_types, d_a) ~ N(0, 1), W1, W3 (d + d_a, h)
    ~ N(0, 1/(d + d_a)), W2 (h, d) ~ N(0, 1/h), all float32 with
    bf16-representable values (the producer holds its weights in bf16)."""
    rng = np.random.default_rng(seed)
    k_in = d + d_a
    return dict(
        table=round_to_bf16(rng.standard_normal((n_types, d_a), dtype=np.float32)),
        W1=round_to_bf16((rng.standard_normal((k_in, h)) / math.sqrt(k_in)).astype(np.float32)),
        W3=round_to_bf16((rng.standard_normal((k_in, h)) / math.sqrt(k_in)).astype(np.float32)),
        W2=round_to_bf16((rng.standard_normal((h, d)) / math.sqrt(h)).astype(np.float32)),
        d=d, d_a=d_a, h=h, n_types=n_types)


def action_types(rows: int, n_types: int, seed: int) -> np.ndarray:
    """Seeded action type ids (rows,) uint8 with P(t) proportional to 2^-t:
    a few common feedback types (a swipe, a finish) and rarer strong ones (a
    like, a follow).  The frequencies are invented; the page names the types
    and gives no mix."""
    rng = np.random.default_rng(seed)
    p = 0.5 ** np.arange(n_types)
    return rng.choice(n_types, size=rows, p=p / p.sum()).astype(np.uint8)
