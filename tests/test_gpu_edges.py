"""GPU edge cases: ragged tails around the 128-row tile, empty users and
batches, k not a multiple of 16, every (d, k) kernel variant, padding
isolation, determinism, additivity, stability, bad offsets and the
host-buffer path.  All through the C ABI, all against the oracle."""

import math

import numpy as np
import pytest

from gpu_util import (TOL, assert_total_mass, assert_user_close, run_gpu, to_device)
from oracle import sa_batch
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu

RAGGED = [1, 127, 128, 129, 0, 300, 255, 2, 1000, 0, 77]


def _full_parity(inp):
    Xt_g, m_g, flags = run_gpu(inp)
    assert flags == 0
    Xt_o, m_o = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                         inp["scale"])
    for b in range(len(inp["offsets"]) - 1):
        assert_user_close(Xt_g[b], m_g[b], Xt_o[b], m_o[b], inp["dtype"], f"user {b}")
    assert_total_mass(m_g, inp["offsets"], inp["dtype"])
    return Xt_g, m_g


@pytest.mark.parametrize("d,k", [(64, 64), (64, 128), (128, 64), (128, 128), (256, 64),
                                 (128, 5), (128, 100), (64, 1), (128, 33),
                                 (256, 256), (256, 200), (256, 65)])
def test_ragged_tails_bf16(d, k):
    _full_parity(make_inputs(RAGGED, d=d, k=k, dtype="bf16", seed=d * 1000 + k))


@pytest.mark.parametrize("d,k", [(64, 16), (128, 64), (256, 256), (64, 3)])
def test_ragged_tails_fp32(d, k):
    _full_parity(make_inputs(RAGGED, d=d, k=k, dtype="fp32", seed=d * 1000 + k))


def test_many_ctas_many_users_bf16():
    # enough rows that every SM gets a range and users straddle many of them
    rng = np.random.default_rng(3)
    lens = rng.integers(0, 9000, size=60)
    _full_parity(make_inputs(lens, d=128, k=128, dtype="bf16", seed=11))


def test_many_tiny_users_per_cta():
    # More users in a CTA's range than the shared-memory copy of the offsets
    # holds (64 entries), so the segment walkers also read offsets from
    # global memory; the 32-way range search takes three rounds.
    rng = np.random.default_rng(21)
    lens = rng.integers(0, 40, size=12000)
    _full_parity(make_inputs(lens, d=128, k=64, dtype="bf16", seed=21))


def test_one_long_user_split_across_all_ctas():
    _full_parity(make_inputs([200_000], d=128, k=64, dtype="bf16", seed=12))


@pytest.mark.parametrize("d,k,dtype", [(128, 128, "bf16"), (64, 64, "fp32"), (256, 256, "bf16")])
def test_split_users_after_empty_and_full_users(d, k, dtype):
    # Long users split over many CTA ranges, some right after a run of empty
    # users and some right after a non-empty user: the finalize pass picks
    # the first range's partial slot by a range search in the first case and
    # in closed form in the second; every user against the oracle.
    lengths = [3000, 0, 0, 0, 40000, 0, 25000, 1, 0, 30000, 17000, 5, 22000, 0]
    _full_parity(make_inputs(lengths, d=d, k=k, dtype=dtype, seed=d + k + 5))


def test_k1_is_column_sum():
    inp = make_inputs([500, 129, 0, 3], d=128, k=1, dtype="bf16", seed=13)
    Xt_g, m_g, _ = run_gpu(inp)
    offs = inp["offsets"]
    for b in range(4):
        want = inp["X"][offs[b]:offs[b + 1]].astype(np.float64).sum(axis=0)
        np.testing.assert_allclose(Xt_g[b, 0], want, rtol=0, atol=1e-3 * max(1, np.abs(want).max()))
        assert m_g[b, 0] == offs[b + 1] - offs[b]


def test_empty_users_and_empty_batch():
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    inp = make_inputs([0, 0, 0], d=128, k=64, dtype="bf16", seed=14)
    Xt_g, m_g, flags = run_gpu(inp)
    assert flags == 0 and not Xt_g.any() and not m_g.any()
    dev = to_device(make_inputs([5], d=128, k=64, dtype="bf16", seed=15))
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], 0.1)
    X0 = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    off0 = torch.zeros(1, dtype=torch.int64, device="cuda")
    Xt, m = q.forward(X0, off0)
    assert Xt.shape == (0, 64, 128) and m.shape == (0, 64)


def test_padding_rows_do_not_leak():
    """NaN and huge rows in the neighbours leave a user's outputs bitwise
    unchanged (section 3.1: padding must not receive mass)."""
    import torch
    inp = make_inputs([300, 129, 1000, 1, 513], d=128, k=128, dtype="bf16", seed=16)
    clean = run_gpu(inp)
    bad = dict(inp)
    X = inp["X"].copy()
    o = inp["offsets"]
    X[o[1]:o[2]] = np.nan
    X[o[3]:o[4]] = 1e30
    bad["X"] = X
    dirty = run_gpu(bad)
    for b in (0, 2, 4):
        assert np.array_equal(clean[0][b], dirty[0][b]), f"user {b} X~ changed"
        assert np.array_equal(clean[1][b], dirty[1][b]), f"user {b} m changed"
    assert np.isnan(dirty[0][1]).any()


def test_bitwise_deterministic():
    inp = make_inputs([70_000, 3, 40_000, 129], d=128, k=128, dtype="bf16", seed=17)
    a = run_gpu(inp)
    b = run_gpu(inp)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_additivity_split_user():
    """One user vs the same rows given as two users: the sums agree."""
    inp = make_inputs([50_000], d=128, k=64, dtype="bf16", seed=18)
    two = dict(inp)
    two["offsets"] = np.array([0, 20_001, 50_000], dtype=np.int64)
    Xa, ma, _ = run_gpu(inp)
    Xb, mb, _ = run_gpu(two)
    assert_user_close(Xb[0] + Xb[1], mb[0] + mb[1], Xa[0], ma[0], "bf16", "split sum")


def _clear_argmax_rows(inp, margin=20.0):
    """Keeps the rows whose best prototype wins by more than twice a bound on
    the kernel's logit error plus `margin` (natural-log units), re-packing
    the users.  The kernel rounds Q' = P W_Q W_K^T * scale to bf16 (relative
    error 2^-9 per entry), so its logit for row i moves by at most
    2^-9 * scale * sum_f |x_if| |Q_jf|; with the gap above that, both sides
    make the same hard decision and the runner-up weighs below e^-margin."""
    X = inp["X"].astype(np.float64)
    Qp = inp["P"].astype(np.float64) @ inp["W_Q"].astype(np.float64) @ \
        inp["W_K"].astype(np.float64).T
    s = inp["scale"]
    L = (X @ Qp.T) * s
    top2 = np.sort(L, axis=1)[:, -2:]
    bound = 2.0 ** -9 * s * (np.abs(X) @ np.abs(Qp).T).max(axis=1)
    keep = (top2[:, 1] - top2[:, 0]) > 2.0 * bound + margin
    offs = inp["offsets"]
    lens = [int(keep[offs[b]:offs[b + 1]].sum()) for b in range(len(offs) - 1)]
    out = dict(inp)
    out["X"] = np.ascontiguousarray(inp["X"][keep])
    out["offsets"] = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return out, keep.mean()


@pytest.mark.parametrize("d,k", [(128, 100), (128, 300), (256, 200)])
def test_large_logits_match_oracle(d, k):
    """Logits of several thousand (scale = 300): the hard-assignment regime,
    where each behaviour's weight sits on one prototype.  Compared entry by
    entry with the oracle, so a wrong maximum (for example a padded
    prototype winning it, k = 100 and 300 leave padded columns; 300 splits
    the prototypes over a cluster of three CTAs, d = 256 with 200 over a
    pair) moves whole rows between prototypes and fails."""
    raw = make_inputs([3000, 129, 1000], d=d, k=k, dtype="bf16", seed=19 + k, scale=300.0)
    inp, kept = _clear_argmax_rows(raw)
    assert kept > 0.5, f"only {kept:.2f} of the rows have a clear winner"
    Xt_g, m_g, flags = run_gpu(inp)
    assert flags == 0
    Xt_o, m_o = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                         inp["scale"])
    assert np.max(np.abs(inp["X"].astype(np.float64))) > 0
    for b in range(len(inp["offsets"]) - 1):
        assert_user_close(Xt_g[b], m_g[b], Xt_o[b], m_o[b], "bf16", f"user {b}")
    assert_total_mass(m_g, inp["offsets"], "bf16")


@pytest.mark.parametrize("bad,flag", [([5, 10, 20], 1), ([0, 30, 20], 2), ([0, 10, 19], 4)])
def test_bad_offsets_raise_device_flag(bad, flag):
    import torch
    from sketch_attention_compression_b200 import SketchQuery, read_device_status
    inp = make_inputs([10, 10], d=128, k=64, dtype="bf16", seed=20)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    offs = torch.tensor(bad, dtype=torch.int64, device="cuda")
    ws = q.new_workspace(2, 20)
    q.forward(dev["X"], offs, workspace=ws)
    assert read_device_status(ws) & flag
    # the next good call on the same workspace is clean
    Xt, m = q.forward(dev["X"], dev["offsets"], workspace=ws)
    assert read_device_status(ws) == 0


def test_workspace_and_alignment_errors():
    import torch
    from sketch_attention_compression_b200 import SAError, SketchQuery
    from sketch_attention_compression_b200.binding import SA_ERR_INVALID_ARG, SA_ERR_WORKSPACE
    inp = make_inputs([100], d=128, k=64, dtype="bf16", seed=21)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(SAError) as e:
        q.forward(dev["X"], dev["offsets"], workspace=small)
    assert e.value.status == SA_ERR_WORKSPACE
    buf = torch.empty(100 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    Xmis = buf[1:1 + 100 * 128].view(100, 128)  # 2-byte offset: not 16-byte aligned
    with pytest.raises(SAError) as e:
        q.forward(Xmis, dev["offsets"])
    assert e.value.status == SA_ERR_INVALID_ARG


def test_host_path_equals_device_path():
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    inp = make_inputs([4000, 0, 129, 77], d=128, k=128, dtype="bf16", seed=22)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    Xt_d, m_d = q.forward(dev["X"], dev["offsets"])
    Xh = dev["X"].cpu().pin_memory()
    Xt_h, m_h = q.forward_host(Xh, inp["offsets"])
    assert np.array_equal(Xt_h, Xt_d.cpu().numpy()) and np.array_equal(m_h, m_d.cpu().numpy())
    from sketch_attention_compression_b200 import SAError
    with pytest.raises(SAError):
        q.forward_host(Xh, np.array([0, 10, 5, 4206, 4206], dtype=np.int64))


def test_partials_then_finalize_equals_forward():
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    inp = make_inputs([90_000, 10, 30_000], d=128, k=64, dtype="bf16", seed=23)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    Xt, m = q.forward(dev["X"], dev["offsets"])
    Xt2 = torch.full_like(Xt, 7.0)
    m2 = torch.full_like(m, 7.0)
    ws = q.new_workspace(3, dev["X"].shape[0])
    q.partials(dev["X"], dev["offsets"], Xt2, m2, ws)
    q.finalize(dev["X"], dev["offsets"], Xt2, m2, ws)
    assert torch.equal(Xt, Xt2) and torch.equal(m, m2)


@pytest.mark.parametrize("d,k,dtype,status", [(256, 257, "bf16", "unsupported"),
                                               (128, 257, "fp32", "unsupported"),
                                               (128, 1025, "bf16", "invalid")])
def test_prototype_limits(d, k, dtype, status):
    """bf16 takes k <= 1024 at d = 64 and 128 (clusters) and k <= 256 at
    d = 256 (pairs); fp32 takes k <= 256.  Beyond: an error on the host."""
    from sketch_attention_compression_b200 import SAError, SketchQuery
    from sketch_attention_compression_b200.binding import SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED
    dev = to_device(make_inputs([10], d=d, k=k, dtype=dtype, seed=24))
    with pytest.raises(SAError) as e:
        SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], 0.1)
    assert e.value.status == (SA_ERR_UNSUPPORTED if status == "unsupported" else SA_ERR_INVALID_ARG)
