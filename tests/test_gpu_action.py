"""GPU parity of the action-fusion producer (section 2.2 "Stacked Refinement
与动作侧融合" of the SequenceO1 reading notes) against the oracle
(oracle/sa_action.py), through the C ABI.

* sa_action_fuse: ragged row counts (one row, a tail of one tile, several
  pairs of tiles per CTA), d = 64 and 128, hidden widths from one chunk
  (64) to eight (512), 1 to 16 action types, action widths 7 to 128;
* an out-of-range type id raises SA_DEVFLAG_ACTION_TYPE and adds no action
  term;
* sa_action_sketch_forward (producer + SA layer) against the SA oracle run
  on the oracle's X rounded to bf16 (the producer's output type), at k = 64
  and on a cluster (k = 300);
* the 16 x 100K history of the benchmark, sampled rows and two users.

Bar for X, element by element, from the arithmetic the kernel does: bf16
operands with exact products and fp32 sums; the per-type rows table W[d:]
rounded to bf16 (2^-9 of |T|); sigma from tanh.approx (absolute error below
2^-12); the gated hidden and X rounded to bf16 (2^-9 each).  With every
rounding term doubled for slack:

  |dx_c| <= 2^-8 |x_c| + sum_k (2^-8 |g_k| + 2^-11 |u_k v_k|
                                + 2^-8 (1.1 |v_k| |T1_k| + |SiLU(u_k)| |T3_k|)) |W2_kc|
            + 1e-5 sum_k |g_k W2_kc|
"""

import numpy as np
import pytest

from gpu_util import assert_total_mass, assert_user_close
from oracle import sa_batch
from oracle.sa_action import action_fuse, fusion_hidden, fusion_input
from oracle.sa_refine import silu
from synthetic import action_params, action_types, generate
from synthetic.workloads import make_inputs, round_to_bf16

pytestmark = pytest.mark.gpu


def _producer(p):
    import torch
    from sketch_attention_compression_b200 import ActionFusion
    t = {key: torch.from_numpy(np.ascontiguousarray(p[key])).cuda()
         for key in ("W1", "W3", "W2", "table")}
    return ActionFusion(t["W1"], t["W3"], t["W2"], t["table"])


def _check_rows(X_gpu, E, types, p, what):
    d = p["d"]
    U, V, G = fusion_hidden(fusion_input(E, types, p["table"]), p["W1"], p["W3"])
    want = np.asarray(E, np.float64) + G @ p["W2"].astype(np.float64)
    T1 = (p["table"].astype(np.float64) @ p["W1"][d:].astype(np.float64))[types]
    T3 = (p["table"].astype(np.float64) @ p["W3"][d:].astype(np.float64))[types]
    aW2 = np.abs(p["W2"].astype(np.float64))
    per_k = (2.0 ** -8 * np.abs(G) + 2.0 ** -11 * np.abs(U * V)
             + 2.0 ** -8 * (1.1 * np.abs(V) * np.abs(T1) + np.abs(silu(U)) * np.abs(T3)))
    bound = 2.0 ** -8 * np.abs(want) + per_k @ aW2 + 1e-5 * (np.abs(G) @ aW2)
    err = np.abs(X_gpu - want)
    assert np.all(np.isfinite(X_gpu)), f"{what}: non-finite"
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (f"{what}: err {err[worst]:.3e} > bound {bound[worst]:.3e} "
                                  f"at {worst}")


@pytest.mark.parametrize("d,d_a,h,n_types,rows", [
    (128, 128, 512, 4, 300), (128, 16, 64, 1, 129), (64, 64, 192, 16, 1000),
    (128, 128, 512, 4, 40000), (64, 7, 128, 5, 1), (128, 32, 256, 16, 77)])
def test_action_fuse_matches_oracle(d, d_a, h, n_types, rows):
    import torch
    inp = make_inputs([rows], d, 16, "bf16", seed=rows + h)
    E = inp["X"]
    types = action_types(rows, n_types, seed=rows)
    p = action_params(d, d_a, h, n_types, seed=d + h + n_types)
    act = _producer(p)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    X = act.fuse(torch.from_numpy(E).cuda().to(torch.bfloat16), torch.from_numpy(types).cuda(),
                 device_flags=flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    _check_rows(X.double().cpu().numpy(), E, types, p, f"rows={rows}")
    act.close()


def test_bad_action_type_is_flagged_and_adds_nothing():
    import torch
    from sketch_attention_compression_b200.binding import DEVFLAG_ACTION_TYPE
    d, d_a, h, n_types, rows = 128, 32, 128, 3, 200
    E = make_inputs([rows], d, 16, "bf16", seed=5)["X"]
    types = action_types(rows, n_types, seed=6)
    types[[0, 77, 199]] = [3, 200, 16]  # outside the table
    p = action_params(d, d_a, h, n_types, seed=7)
    act = _producer(p)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    X = act.fuse(torch.from_numpy(E).cuda().to(torch.bfloat16), torch.from_numpy(types).cuda(),
                 device_flags=flags)
    torch.cuda.synchronize()
    assert flags.item() & DEVFLAG_ACTION_TYPE
    # Expected: the bad rows see a zero action embedding.
    q = dict(p)
    q["table"] = np.vstack([p["table"], np.zeros((1, d_a), np.float32)])
    fixed = np.where(types < n_types, types, n_types)
    _check_rows(X.double().cpu().numpy(), E, fixed, q, "bad types")
    act.close()


def _query(inp):
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    t = {key: torch.from_numpy(inp[key]).cuda().to(torch.bfloat16) for key in ("P", "W_Q", "W_K")}
    return SketchQuery(t["P"], t["W_Q"], t["W_K"], inp["scale"])


def _sketch_parity(inp, types, p, users):
    import torch
    from sketch_attention_compression_b200 import read_device_status
    act = _producer(p)
    q = _query(inp)
    E = torch.from_numpy(inp["X"]).cuda().to(torch.bfloat16)
    offs = torch.from_numpy(inp["offsets"]).cuda()
    Xt, m, ws = act.sketch_forward(q, E, torch.from_numpy(types).cuda(), offs)
    assert read_device_status(ws) == 0
    Xg, mg = Xt.double().cpu().numpy(), m.double().cpu().numpy()
    off = inp["offsets"]
    for b in users:
        lo, hi = int(off[b]), int(off[b + 1])
        Xo = round_to_bf16(action_fuse(inp["X"][lo:hi], types[lo:hi], p["table"], p["W1"], p["W3"],
                                       p["W2"]).astype(np.float32))
        xs, ms = sa_batch(Xo, [0, hi - lo], inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
        assert_user_close(Xg[b], mg[b], xs[0], ms[0], "bf16", f"user {b}")
    assert_total_mass(mg, off, "bf16")
    act.close()
    q.close()


@pytest.mark.parametrize("k", [64, 300])
def test_action_sketch_forward_matches_oracle(k):
    lengths = [700, 0, 129, 3000, 1, 255, 4100, 96]
    inp = make_inputs(lengths, 128, k, "bf16", seed=k + 1)
    types = action_types(int(inp["offsets"][-1]), 4, seed=k)
    p = action_params(128, 128, 512, 4, seed=k + 2)
    _sketch_parity(inp, types, p, range(len(lengths)))


def test_action_full_size_sampled():
    """The benchmark's 16 x 100K history, h = 512, four action types: a
    sample of producer rows, and two users through producer + SA."""
    import torch
    inp = generate("batch16_n100k_d128_k128_mixture_bf16")
    N = int(inp["offsets"][-1])
    types = action_types(N, 4, seed=11)
    p = action_params(128, 128, 512, 4, seed=12)
    act = _producer(p)
    E = torch.from_numpy(inp["X"]).cuda().to(torch.bfloat16)
    X = act.fuse(E, torch.from_numpy(types).cuda())
    rng = np.random.default_rng(13)
    rows = np.unique(np.concatenate([rng.integers(0, N, 3000), np.arange(N - 200, N)]))
    _check_rows(X[torch.from_numpy(rows).cuda()].double().cpu().numpy(), inp["X"][rows],
                types[rows], p, "full size")
    act.close()
    _sketch_parity(inp, types, p, [0, 15])
