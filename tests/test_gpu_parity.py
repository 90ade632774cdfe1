"""GPU parity: the CUDA path against the CPU oracle on the five seeded
workloads, at their full sizes, in the launch configuration the benchmark
uses.  Where the oracle would take too long for every user, a fixed sample
of users is compared entry by entry and every user is checked against the
closed form sum_j m_j = n_b."""

import numpy as np
import pytest

from gpu_util import assert_total_mass, assert_user_close, run_gpu
from oracle import sa_batch
from synthetic import generate

pytestmark = pytest.mark.gpu


def _parity(name, users=None):
    inp = generate(name)
    Xt_g, m_g, flags = run_gpu(inp)
    assert flags == 0
    B = len(inp["offsets"]) - 1
    sel = list(range(B)) if users is None else users(inp)
    Xt_o, m_o = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                         inp["scale"], users=sel)
    worst = (0.0, 0.0)
    for b in sel:
        ex, em = assert_user_close(Xt_g[b], m_g[b], Xt_o[b], m_o[b], inp["dtype"], f"user {b}")
        worst = (max(worst[0], ex), max(worst[1], em))
    assert_total_mass(m_g, inp["offsets"], inp["dtype"])
    return worst


def test_single_user_fp32():
    _parity("single_n1024_d64_k16_fp32")


def test_batch32_n10k_d128_k64():
    _parity("batch32_n10k_d128_k64_bf16")


def test_batch16_n100k_d128_k128_mixture():
    _parity("batch16_n100k_d128_k128_mixture_bf16", users=lambda inp: [0, 7, 15])


def test_ragged256_d128_k64():
    def pick(inp):
        n = np.diff(inp["offsets"])
        return sorted({int(np.argmin(n)), int(np.argmax(n)), 0, 100, 255})
    _parity("ragged256_loguniform_1k_100k_d128_k64_bf16", users=pick)


def test_batch8_n100k_d256_k256():
    _parity("batch8_n100k_d256_k256_bf16", users=lambda inp: [0, 7])
