"""GPU parity of per-user queries (the SA step of a refinement layer,
section 2.2 "Stacked Refinement" of the SequenceO1 reading notes): user b's
rows queried by its own Q_b, through sa_sketch_forward_user_queries, against
the oracle's sa_batch_user_queries on the same seeded inputs."""

import ctypes

import numpy as np
import pytest

from gpu_util import assert_total_mass, assert_user_close, to_device
from oracle import sa_batch, sa_batch_user_queries, mass_normalised
from synthetic import generate, user_queries
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu

RAGGED = [1, 127, 128, 129, 0, 300, 255, 2, 1000, 0, 77]


def _run_gpu(inp, queries, dev=None):
    import torch
    from sketch_attention_compression_b200 import SketchQuery, read_device_status
    dev = to_device(inp) if dev is None else dev
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    Qd = torch.from_numpy(np.ascontiguousarray(queries, dtype=np.float32)).cuda()
    B = len(inp["offsets"]) - 1
    ws = torch.empty(q.workspace_bytes_user_queries(B, dev["X"].shape[0]), dtype=torch.uint8,
                     device="cuda")
    Xt, m = q.forward_user_queries(Qd, dev["X"], dev["offsets"], workspace=ws)
    flags = read_device_status(ws)
    torch.cuda.synchronize()
    out = Xt.double().cpu().numpy(), m.double().cpu().numpy(), flags
    q.close()
    return out


def _parity(inp, queries, users=None):
    Xt_g, m_g, flags = _run_gpu(inp, queries)
    assert flags == 0
    B = len(inp["offsets"]) - 1
    sel = list(range(B)) if users is None else users
    Xt_o, m_o = sa_batch_user_queries(inp["X"], inp["offsets"], queries, inp["W_Q"], inp["W_K"],
                                      inp["scale"], users=sel)
    for b in sel:
        assert_user_close(Xt_g[b], m_g[b], Xt_o[b], m_o[b], inp["dtype"], f"user {b}")
    assert_total_mass(m_g, inp["offsets"], inp["dtype"])
    return Xt_g, m_g


@pytest.mark.parametrize("d,k", [(64, 64), (64, 128), (128, 64), (128, 128), (256, 64),
                                 (128, 5), (128, 100), (64, 1), (128, 33), (256, 200),
                                 (256, 256)])
def test_ragged_tails_bf16(d, k):
    inp = make_inputs(RAGGED, d=d, k=k, dtype="bf16", seed=7 * d + k)
    _parity(inp, user_queries(len(RAGGED), k, d, seed=d + k))


@pytest.mark.parametrize("d,k", [(64, 16), (128, 64), (256, 256), (64, 3)])
def test_ragged_tails_fp32(d, k):
    inp = make_inputs(RAGGED, d=d, k=k, dtype="fp32", seed=7 * d + k)
    _parity(inp, user_queries(len(RAGGED), k, d, seed=d + k))


@pytest.mark.parametrize("d,k,users", [(128, 128, 3000), (256, 256, 1200)])
def test_many_users_per_cta_reload_queries(d, k, users):
    # Thousands of short users: every CTA (or CTA pair) reloads Q' dozens of
    # times, and users cross CTA ranges.
    rng = np.random.default_rng(31)
    lens = rng.integers(0, 400, size=users)
    inp = make_inputs(lens, d=d, k=k, dtype="bf16", seed=31)
    _parity(inp, user_queries(len(lens), k, d, seed=31))


def test_long_user_split_across_ctas():
    lens = [200_000, 5, 0, 3000]
    inp = make_inputs(lens, d=128, k=64, dtype="bf16", seed=32)
    _parity(inp, user_queries(len(lens), 64, 128, seed=32))


def test_batch16_n100k_d128_k128_sampled():
    # The 16 x 100K mixture batch at d = k = 128 with per-user queries:
    # three users entry by entry, every user by its total mass.
    inp = generate("batch16_n100k_d128_k128_mixture_bf16")
    _parity(inp, user_queries(16, 128, 128, seed=1102), users=[0, 7, 15])


def test_only_own_queries_matter():
    # Changing user 1's queries leaves every other user's outputs bitwise
    # unchanged and changes user 1's.
    inp = make_inputs([700, 300, 0, 900], d=128, k=64, dtype="bf16", seed=33)
    Q = user_queries(4, 64, 128, seed=33)
    Xt_a, m_a, _ = _run_gpu(inp, Q)
    Q2 = Q.copy()
    Q2[1] = -2.0 * Q2[1]
    Xt_b, m_b, _ = _run_gpu(inp, Q2)
    for b in (0, 2, 3):
        assert np.array_equal(Xt_a[b], Xt_b[b]) and np.array_equal(m_a[b], m_b[b])
    assert not np.allclose(Xt_a[1], Xt_b[1])
    assert np.all(Xt_a[2] == 0) and np.all(m_a[2] == 0)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_two_stacked_layers(dtype):
    # Layer 1 queries with the shared prototypes, layer 2 with the layer-1
    # sketch normalised by its masses (X~_j / m_j); each side runs its own
    # chain and the final sketches are compared.
    import torch
    from sketch_attention_compression_b200 import SketchQuery, mass_normalise
    lens = [3000, 129, 0, 5000, 64]
    d, k = 128, 64
    inp = make_inputs(lens, d=d, k=k, dtype=dtype, seed=34)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    Xt1, m1 = q.forward(dev["X"], dev["offsets"])
    Q2 = mass_normalise(Xt1, m1)
    Xt2, m2 = q.forward_user_queries(Q2, dev["X"], dev["offsets"])
    torch.cuda.synchronize()
    Xt_g, m_g = Xt2.double().cpu().numpy(), m2.double().cpu().numpy()
    q.close()
    Xt1_o, m1_o = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                           inp["scale"])
    Q2_o = np.stack([mass_normalised(Xt1_o[b], m1_o[b]) for b in range(len(lens))])
    Xt_o, m_o = sa_batch_user_queries(inp["X"], inp["offsets"], Q2_o, inp["W_Q"], inp["W_K"],
                                      inp["scale"])
    for b in range(len(lens)):
        assert_user_close(Xt_g[b], m_g[b], Xt_o[b], m_o[b], dtype, f"user {b}")
    assert_total_mass(m_g, inp["offsets"], dtype)


def test_errors():
    import torch
    from sketch_attention_compression_b200 import SketchQuery, binding
    inp = make_inputs([300, 10], d=128, k=64, dtype="bf16", seed=36)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    Qd = torch.zeros((2, 64, 128), dtype=torch.float32, device="cuda")
    small = torch.empty(q.workspace_bytes(2, 310), dtype=torch.uint8, device="cuda")
    assert q.workspace_bytes_user_queries(2, 310) > q.workspace_bytes(2, 310)
    with pytest.raises(binding.SAError) as e:
        q.forward_user_queries(Qd, dev["X"], dev["offsets"], workspace=small)
    assert e.value.status == binding.SA_ERR_WORKSPACE
    Xt = torch.empty((2, 64, 128), dtype=torch.float32, device="cuda")
    m = torch.empty((2, 64), dtype=torch.float32, device="cuda")
    ws = torch.empty(q.workspace_bytes_user_queries(2, 310), dtype=torch.uint8, device="cuda")
    st = q._lib.sa_sketch_forward_user_queries(
        q._h, ctypes.c_void_p(0), ctypes.c_void_p(dev["X"].data_ptr()),
        ctypes.c_void_p(dev["offsets"].data_ptr()), 2, 310, ctypes.c_void_p(Xt.data_ptr()),
        ctypes.c_void_p(m.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
        ctypes.c_void_p(0))
    assert st == binding.SA_ERR_INVALID_ARG
    q.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_queries_only_4_byte_aligned(dtype):
    # The Q'_b kernel stages 16-byte units of Q when the array is 16-byte
    # aligned and single words otherwise; both give the same sketches, bit
    # for bit, and match the oracle.
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    lengths = [300, 129, 1, 0, 700]
    inp = make_inputs(lengths, d=128, k=100, dtype=dtype, seed=41)
    queries = user_queries(len(lengths), 100, 128, seed=42)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    flat = torch.from_numpy(queries.astype(np.float32).ravel()).cuda()
    buf = torch.zeros(flat.numel() + 4, dtype=torch.float32, device="cuda")
    buf[1:1 + flat.numel()] = flat
    shape = (len(lengths), 100, 128)
    Q16, Q4 = flat.view(shape), buf[1:1 + flat.numel()].view(shape)
    assert Q16.data_ptr() % 16 == 0 and Q4.data_ptr() % 16 == 4
    outs = []
    for Qd in (Q16, Q4):
        Xt, m = q.forward_user_queries(Qd, dev["X"], dev["offsets"], check=True)
        outs.append((Xt.cpu(), m.cpu()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    q.close()
    Xt_o, m_o = sa_batch_user_queries(inp["X"], inp["offsets"], queries, inp["W_Q"], inp["W_K"],
                                      inp["scale"])
    for b in range(len(lengths)):
        assert_user_close(outs[1][0][b].double().numpy(), outs[1][1][b].double().numpy(),
                          Xt_o[b], m_o[b], dtype, f"user {b}")


def test_mass_normalise():
    # X~_j / m_j against the oracle's mass_normalised, 0 for the empty
    # user's rows; in place gives the same bits.
    import torch
    from sketch_attention_compression_b200 import SketchQuery, mass_normalise
    lens = [700, 0, 1, 2500]
    inp = make_inputs(lens, d=128, k=100, dtype="bf16", seed=37)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    Xt, m = q.forward(dev["X"], dev["offsets"])
    out = mass_normalise(Xt, m)
    torch.cuda.synchronize()
    Xn = out.double().cpu().numpy()
    Xt_o, m_o = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
    for b in range(len(lens)):
        ref = mass_normalised(Xt_o[b], m_o[b])
        assert np.max(np.abs(Xn[b] - ref)) <= 2e-2 * max(np.max(np.abs(ref)), 1e-30), f"user {b}"
    assert np.all(Xn[1] == 0)
    # the kernel divides the library's own X~ by its own m: compare with fp32 division
    want = torch.where(m[..., None] > 0, Xt / m[..., None], torch.zeros_like(Xt))
    assert torch.equal(out, want)
    Xt2 = Xt.clone()
    mass_normalise(Xt2, m, out=Xt2)
    assert torch.equal(Xt2, out)
    q.close()
