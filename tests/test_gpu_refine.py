"""GPU parity of the stacked refinement layers (section 2.2 "Stacked
Refinement" of the SequenceO1 reading notes) against the oracle
(oracle/sa_refine.py), through the C ABI.

* sa_refine_update alone: ragged tails of the 128-row tiles, d = 64 and 128,
  hidden widths 128 and 512, shared and per-user residuals, empty prototypes;
* sa_refine_layer_forward: layer 1 (queried by P) and layer 2 (per-user
  queries from layer 1) at k = 64, 128 and 300 (a cluster of three CTAs);
* sa_refine_stack_forward: the final configuration of the notes, two layers
  at k = 1000 and d = 128, on clusters of eight CTAs;
* device flags: a bad offsets array is reported after a stacked call.

Bar (tests/test_refine_arithmetic.py emulates the kernel's rounding points at
about 8x inside it): per user, max |out - oracle| <= 2e-2 * max |oracle|.
"""

import numpy as np
import pytest

from gpu_util import to_device
from oracle import refine_layer, refine_stack, refine_update
from synthetic import refine_params
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _close_users(got, want, what):
    for b in range(want.shape[0]):
        ref = np.abs(want[b]).max()
        err = np.abs(got[b] - want[b]).max()
        assert np.all(np.isfinite(got[b])), f"{what} user {b}: non-finite"
        assert err <= TOL * ref, f"{what} user {b}: err {err:.3e} > {TOL} * {ref:.3e}"


def _refine_handle(p):
    import torch
    from sketch_attention_compression_b200 import RefineParams
    t = {key: torch.from_numpy(np.ascontiguousarray(p[key])).cuda()
         for key in ("W1", "W3", "W2", "gamma1", "beta1", "gamma2", "beta2")}
    return RefineParams(t["W1"], t["W3"], t["W2"], t["gamma1"], t["beta1"], t["gamma2"],
                        t["beta2"])


def _query(P, p):
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    return SketchQuery(torch.from_numpy(P).cuda().to(torch.bfloat16),
                       torch.from_numpy(p["W_Q"]).cuda().to(torch.bfloat16),
                       torch.from_numpy(p["W_K"]).cuda().to(torch.bfloat16), p["scale"])


@pytest.mark.parametrize("d,h,shared", [(128, 512, False), (128, 128, True), (64, 256, False),
                                        (64, 128, True)])
def test_refine_update_matches_oracle(d, h, shared):
    import torch
    rng = np.random.default_rng(d * 7 + h)
    B, k = 3, 100  # 300 rows: two full tiles and a tail of 44
    prev = rng.standard_normal((k, d) if shared else (B, k, d)).astype(np.float32)
    m = rng.uniform(0.0, 500.0, (B, k)).astype(np.float32)
    m[0, :5] = 0.0
    m[2, 50:] = 0.0
    Xt = (rng.standard_normal((B, k, d)) * 0.3 * m[..., None]).astype(np.float32)
    p = refine_params(d, h, seed=d + h)
    r = _refine_handle(p)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = r.update(torch.from_numpy(prev).cuda(), torch.from_numpy(Xt).cuda(),
                   torch.from_numpy(m).cuda(), prev_shared=shared, device_flags=flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    want = refine_update(np.broadcast_to(prev, (B, k, d)) if shared else prev, Xt, m, p)
    _close_users(out.double().cpu().numpy(), want, "update")
    r.close()


@pytest.mark.parametrize("k", [64, 128, 300])
def test_refine_layers_one_and_two(k):
    import torch
    from sketch_attention_compression_b200 import read_device_status, refine_layer_forward
    d, h = 128, 512
    inp = make_inputs([3000, 0, 129, 1000], d=d, k=k, dtype="bf16", seed=70 + k)
    dev = to_device(inp)
    P32 = torch.from_numpy(inp["P"]).cuda()
    layers = [refine_params(d, h, seed=80 + k), refine_params(d, h, seed=90 + k)]
    qs = [_query(inp["P"], L) for L in layers]
    rs = [_refine_handle(L) for L in layers]
    out1, ws = refine_layer_forward(qs[0], rs[0], dev["X"], dev["offsets"], P_f32=P32)
    assert read_device_status(ws) == 0
    want1 = refine_layer(inp["X"], inp["offsets"], None, inp["P"], layers[0])
    got1 = out1.double().cpu().numpy()
    _close_users(got1, want1, "layer 1")
    # layer 2 queried by the GPU's own layer-1 output (isolates layer 2)
    out2, ws = refine_layer_forward(qs[1], rs[1], dev["X"], dev["offsets"], prev=out1)
    assert read_device_status(ws) == 0
    want2 = refine_layer(inp["X"], inp["offsets"], got1, inp["P"], layers[1])
    _close_users(out2.double().cpu().numpy(), want2, "layer 2")
    for o in qs + rs:
        o.close()


def test_refine_stack_two_layers_k1000():
    """Two layers, about a thousand prototypes, width 128 (the final
    configuration of section 2.2), against the oracle's whole stack."""
    import torch
    from sketch_attention_compression_b200 import read_device_status, refine_stack_forward
    d, h, k = 128, 512, 1000
    inp = make_inputs([6000, 129, 0, 2500], d=d, k=k, dtype="bf16", seed=101,
                      x_kind="mixture")
    dev = to_device(inp)
    layers = [refine_params(d, h, seed=111), refine_params(d, h, seed=112)]
    qs = [_query(inp["P"], L) for L in layers]
    rs = [_refine_handle(L) for L in layers]
    out, ws = refine_stack_forward(qs, rs, torch.from_numpy(inp["P"]).cuda(), dev["X"],
                                   dev["offsets"])
    assert read_device_status(ws) == 0
    want = refine_stack(inp["X"], inp["offsets"], inp["P"], layers)
    _close_users(out.double().cpu().numpy(), want, "stack")
    for o in qs + rs:
        o.close()


def test_refine_stack_full_size_sampled():
    # Two layers at k = 1000 on the benchmark's 16 x 100K workload, in the
    # benchmark's launch configuration; a user's stack depends on its own
    # rows only, so users 0 and 15 are checked against the oracle's stack
    # (about four seconds each on the CPU).
    import torch
    from sketch_attention_compression_b200 import read_device_status, refine_stack_forward
    from synthetic import generate
    inp = generate("batch16_n100k_d128_k1000_mixture_bf16")
    d, h = 128, 512
    layers = [refine_params(d, h, seed=321), refine_params(d, h, seed=322)]
    dev = to_device(inp)
    qs = [_query(inp["P"], L) for L in layers]
    rs = [_refine_handle(L) for L in layers]
    out, ws = refine_stack_forward(qs, rs, torch.from_numpy(inp["P"]).cuda(), dev["X"],
                                   dev["offsets"])
    assert read_device_status(ws) == 0
    users = [0, 15]
    want = refine_stack(inp["X"], inp["offsets"], inp["P"], layers, users=users)
    _close_users(out.double().cpu().numpy()[users], want[users], "full-size stack")
    for o in qs + rs:
        o.close()


def test_refine_stack_reports_bad_offsets():
    import torch
    from sketch_attention_compression_b200 import read_device_status, refine_stack_forward
    d, h, k = 128, 128, 64
    inp = make_inputs([500, 300], d=d, k=k, dtype="bf16", seed=121)
    dev = to_device(inp)
    layers = [refine_params(d, h, seed=122), refine_params(d, h, seed=123)]
    qs = [_query(inp["P"], L) for L in layers]
    rs = [_refine_handle(L) for L in layers]
    bad = torch.tensor([0, 500, 799], dtype=torch.int64, device="cuda")  # N is 800
    _, ws = refine_stack_forward(qs, rs, torch.from_numpy(inp["P"]).cuda(), dev["X"], bad)
    assert read_device_status(ws) & 4  # SA_DEVFLAG_OFFSET_LAST
    _, ws2 = refine_stack_forward(qs, rs, torch.from_numpy(inp["P"]).cuda(), dev["X"],
                                  dev["offsets"], workspace=ws)
    assert read_device_status(ws2) == 0
    for o in qs + rs:
        o.close()
