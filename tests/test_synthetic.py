"""The seeded input generators: determinism, shapes, bf16 rounding."""

import math

import numpy as np
import pytest

from synthetic import WORKLOADS, bf16_bits, bf16_from_bits, generate, round_to_bf16
from synthetic.workloads import make_inputs, ragged_lengths


def test_bf16_round_to_nearest_even():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -7)  # bf16 spacing at 1.0
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -20,
                  -2.5, 65504.0, 3.0e38], dtype=np.float32)
    r = round_to_bf16(x)
    assert r[0] == one
    assert r[1] == one                       # tie -> even (mantissa 0)
    assert r[2] == one + 2 * ulp             # tie -> even (mantissa 2)
    assert r[3] == one + ulp                 # above the tie -> up
    assert r[4] == np.float32(-2.5)
    assert np.all(bf16_from_bits(bf16_bits(r)) == r)  # idempotent
    assert bf16_bits(np.array([np.nan], np.float32))[0] & 0x7FFF == 0x7FC0
    assert np.isinf(round_to_bf16(np.array([np.inf], np.float32)))[0]


def test_make_inputs_deterministic_and_shaped():
    a = make_inputs([3, 0, 4], d=8, k=5, dtype="bf16", seed=3)
    b = make_inputs([3, 0, 4], d=8, k=5, dtype="bf16", seed=3)
    for key in ("X", "P", "W_Q", "W_K", "offsets"):
        assert np.array_equal(a[key], b[key])
    assert a["X"].shape == (7, 8) and a["P"].shape == (5, 8)
    assert a["W_Q"].shape == (8, 8) and list(a["offsets"]) == [0, 3, 3, 7]
    assert np.all(round_to_bf16(a["X"]) == a["X"])
    assert a["scale"] == pytest.approx(1 / math.sqrt(8))


def test_ragged_lengths_in_range():
    rng = np.random.default_rng(0)
    n = ragged_lengths(rng, 5000, 1000, 100000)
    assert n.min() >= 1000 and n.max() < 100000
    # log-uniform: the median is near the geometric mean of the bounds
    assert 7000 < np.median(n) < 13000


def test_workload_table():
    assert len(WORKLOADS) == 6
    w = WORKLOADS["batch16_n100k_d128_k128_mixture_bf16"]
    assert (w.batch, w.n, w.d, w.k, w.x_kind) == (16, 100_000, 128, 128, "mixture")


def test_small_workload_generation():
    inp = generate("single_n1024_d64_k16_fp32")
    assert inp["X"].dtype == np.float32 and inp["X"].shape == (1024, 64)
    assert list(inp["offsets"]) == [0, 1024]
    # W ~ N(0, 1/d): sample sd near 1/8
    assert abs(inp["W_K"].std() - 1 / 8) < 0.01


def test_workload_lengths_are_generate_first_draws():
    """workload_lengths (used by the bench to count each rank's rows) draws
    exactly the lengths that generate draws first."""
    import numpy as np
    from synthetic import WORKLOADS, generate, ragged_lengths, workload_lengths
    for name in ("single_n1024_d64_k16_fp32", "batch32_n10k_d128_k64_bf16"):
        assert np.array_equal(workload_lengths(name), np.diff(generate(name)["offsets"]))
        assert np.array_equal(workload_lengths(name, seed=7), np.diff(generate(name, seed=7)["offsets"]))
    w = WORKLOADS["ragged256_loguniform_1k_100k_d128_k64_bf16"]
    want = ragged_lengths(np.random.default_rng(w.seed + 1), w.batch, w.lo, w.hi)
    assert np.array_equal(workload_lengths(w.name, seed=w.seed + 1), want)
