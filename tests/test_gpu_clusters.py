"""GPU parity of the prototype-split clusters: bf16, d = 64 or 128, more
than 128 prototypes (up to 1024; section 2.2 "Stacked Refinement" of the
SequenceO1 reading notes gives about a thousand prototypes for the final
layers).  C = ceil(k / 128) CTAs share each row range, one 128-prototype
slice each, and combine the softmax statistics of every row across the
cluster.  Everything through the C ABI, against the oracle."""

import numpy as np
import pytest

from gpu_util import assert_total_mass, assert_user_close, run_gpu, to_device
from oracle import sa_batch, sa_batch_user_queries
from synthetic import generate, user_queries
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu

RAGGED = [1, 127, 128, 129, 0, 300, 255, 2, 1000, 0, 77]


def _full_parity(inp, users=None):
    Xt_g, m_g, flags = run_gpu(inp)
    assert flags == 0
    B = len(inp["offsets"]) - 1
    sel = list(range(B)) if users is None else users
    Xt_o, m_o = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                         inp["scale"], users=sel)
    for b in sel:
        assert_user_close(Xt_g[b], m_g[b], Xt_o[b], m_o[b], inp["dtype"], f"user {b}")
    assert_total_mass(m_g, inp["offsets"], inp["dtype"])
    return Xt_g, m_g


@pytest.mark.parametrize("d,k", [(128, 129), (128, 200), (128, 256), (128, 300), (128, 512),
                                 (128, 640), (128, 1000), (128, 1024), (64, 256), (64, 1000)])
def test_ragged_tails(d, k):
    _full_parity(make_inputs(RAGGED, d=d, k=k, dtype="bf16", seed=3 * d + k))


def test_many_users_across_cluster_ranges():
    rng = np.random.default_rng(41)
    lens = rng.integers(0, 9000, size=60)
    _full_parity(make_inputs(lens, d=128, k=1000, dtype="bf16", seed=41))


def test_one_long_user_split_across_all_clusters():
    _full_parity(make_inputs([300_000], d=128, k=384, dtype="bf16", seed=42))


def test_per_user_queries_on_clusters():
    lens = [3000, 0, 129, 700, 5000]
    inp = make_inputs(lens, d=128, k=1000, dtype="bf16", seed=43)
    Q = user_queries(len(lens), 1000, 128, seed=43)
    import torch
    from sketch_attention_compression_b200 import SketchQuery, read_device_status
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    ws = torch.empty(q.workspace_bytes_user_queries(len(lens), dev["X"].shape[0]),
                     dtype=torch.uint8, device="cuda")
    Xt, m = q.forward_user_queries(torch.from_numpy(Q).cuda(), dev["X"], dev["offsets"],
                                   workspace=ws)
    assert read_device_status(ws) == 0
    Xt_g, m_g = Xt.double().cpu().numpy(), m.double().cpu().numpy()
    q.close()
    Xt_o, m_o = sa_batch_user_queries(inp["X"], inp["offsets"], Q, inp["W_Q"], inp["W_K"],
                                      inp["scale"])
    for b in range(len(lens)):
        assert_user_close(Xt_g[b], m_g[b], Xt_o[b], m_o[b], "bf16", f"user {b}")
    assert_total_mass(m_g, inp["offsets"], "bf16")


def test_padding_rows_do_not_leak():
    # NaN and huge rows around a user change nothing of its sketch.
    inp = make_inputs([200, 300, 200], d=128, k=600, dtype="bf16", seed=44)
    X2 = inp["X"].copy()
    X2[:200] = np.nan
    X2[500:] = 3e38
    inp2 = dict(inp, X=X2)
    Xt_a, m_a, _ = run_gpu(inp)
    Xt_b, m_b, _ = run_gpu(inp2)
    assert np.array_equal(Xt_a[1], Xt_b[1]) and np.array_equal(m_a[1], m_b[1])


def test_prototype_permutation_across_slices():
    # Reversing the order of 1000 prototypes moves every prototype to
    # another CTA's slice; the sketch rows must follow (section 2.1: the
    # softmax runs over the whole prototype axis).
    inp = make_inputs([4000, 129, 3], d=128, k=1000, dtype="bf16", seed=45)
    rev = dict(inp, P=np.ascontiguousarray(inp["P"][::-1]))
    Xt_a, m_a, _ = run_gpu(inp)
    Xt_b, m_b, _ = run_gpu(rev)
    for b in range(3):
        assert_user_close(Xt_b[b][::-1], m_b[b][::-1], Xt_a[b], m_a[b], "bf16", f"user {b}")


def test_bitwise_deterministic():
    inp = make_inputs([40_000, 7, 900], d=128, k=1000, dtype="bf16", seed=46)
    dev = to_device(inp)
    a = run_gpu(inp, dev)
    b = run_gpu(inp, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_batch16_n100k_d128_k1000_sampled():
    # The 16 x 100K mixture batch with the final layers' prototype count:
    # users 0 and 15 entry by entry, every user by its total mass.
    _full_parity(generate("batch16_n100k_d128_k1000_mixture_bf16"), users=[0, 15])
