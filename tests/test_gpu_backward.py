"""GPU parity of the SA backward pass (sa_sketch_backward) against the
gradient oracle (oracle/sa_backward.py, pinned by finite differences), through
the C ABI.

Section 2.2 of the SequenceO1 reading notes trains the module end to end;
the gradients are the chain rule through section 2.1's forward.  Cases:
ragged tails around the 128-row tile, empty users, padded prototypes
(k = 100, 33), d = 64 and 128, the mass gradient g present or absent, shared
prototypes (dP summed over users) and per-user queries (dQ_b), a user split
across every CTA (partial R summed in a fixed order), bitwise determinism.

Bar (a CPU emulation of the kernel's rounding points lands near 4e-3):
dX per user max |err| <= 2e-2 * max |oracle dX of that user|; dP (or each
dQ_b), dW_Q, dW_K likewise against their own maxima.
"""

import numpy as np
import pytest

from gpu_util import to_device
from oracle.sa_backward import sa_batch_backward
from synthetic import upstream_gradients, user_queries
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _close(got, want, what):
    ref = np.abs(want).max()
    err = np.abs(got - want).max()
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    assert err <= TOL * max(ref, 1e-30), f"{what}: err {err:.3e} > {TOL} * {ref:.3e}"


def _run(inp, per_user, with_g, seed):
    import torch
    from sketch_attention_compression_b200 import SketchQuery, read_device_status
    dev = to_device(inp)
    B = len(inp["offsets"]) - 1
    k, d = inp["P"].shape
    G, g = upstream_gradients(B, k, d, seed)
    G = G.astype(np.float32)
    g = g.astype(np.float32) if with_g else None
    Q = user_queries(B, k, d, seed + 1) if per_user else None
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()  # noqa: E731
    out, ws = q.backward(dev["X"], dev["offsets"], f32(G), None if g is None else f32(g),
                         P_f32=f32(inp["P"]), W_Q_f32=f32(inp["W_Q"]), W_K_f32=f32(inp["W_K"]),
                         queries=None if Q is None else f32(Q))
    assert read_device_status(ws) == 0
    got = {key: v.double().cpu().numpy() for key, v in out.items()}
    q.close()
    want = sa_batch_backward(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                             inp["scale"], G, g, queries=Q)
    return got, want


def _check(got, want, offsets):
    for b in range(len(offsets) - 1):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        if hi > lo:
            _close(got["dX"][lo:hi], want["dX"][lo:hi], f"dX user {b}")
    if "dP" in want:
        _close(got["dP"], want["dP"], "dP")
    else:
        for b in range(len(offsets) - 1):
            if offsets[b + 1] > offsets[b]:
                _close(got["dQueries"][b], want["dQueries"][b], f"dQ user {b}")
            else:
                assert not got["dQueries"][b].any(), f"empty user {b} has a query gradient"
    _close(got["dW_Q"], want["dW_Q"], "dW_Q")
    _close(got["dW_K"], want["dW_K"], "dW_K")


RAGGED = [1000, 0, 129, 300, 1, 128]


@pytest.mark.parametrize("d,k,per_user,with_g", [(128, 128, False, True), (128, 64, False, True),
                                                 (64, 64, False, False), (128, 100, False, True),
                                                 (128, 128, True, True), (64, 33, True, False),
                                                 (64, 128, True, True)])
def test_backward_matches_oracle(d, k, per_user, with_g):
    inp = make_inputs(RAGGED, d=d, k=k, dtype="bf16", seed=200 + d + k)
    got, want = _run(inp, per_user, with_g, seed=300 + k)
    _check(got, want, inp["offsets"])


def test_backward_user_split_across_all_ctas():
    inp = make_inputs([100_000], d=128, k=64, dtype="bf16", seed=210)
    got, want = _run(inp, per_user=False, with_g=True, seed=310)
    _check(got, want, inp["offsets"])


def test_backward_full_size_benchmark_workload():
    # The benchmark's workload and launch configuration (16 users x 100K
    # rows, d = k = 128, mixture X, G and g ~ N(0, 1)); every output of every
    # user against the oracle (about half a second per user on the CPU).
    from synthetic import generate
    inp = generate("batch16_n100k_d128_k128_mixture_bf16")
    got, want = _run(inp, per_user=False, with_g=True, seed=330)
    _check(got, want, inp["offsets"])


def test_backward_bitwise_deterministic():
    inp = make_inputs([40_000, 3, 20_000], d=128, k=128, dtype="bf16", seed=220, x_kind="mixture")
    a, _ = _run(inp, per_user=False, with_g=True, seed=320)
    b, _ = _run(inp, per_user=False, with_g=True, seed=320)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


def test_backward_unsupported_shapes_are_refused():
    import torch
    from sketch_attention_compression_b200 import SAError, SketchQuery
    from sketch_attention_compression_b200.binding import SA_ERR_UNSUPPORTED
    for d, k in [(256, 64), (128, 200)]:
        inp = make_inputs([10], d=d, k=k, dtype="bf16", seed=230)
        dev = to_device(inp)
        q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
        G = torch.zeros((1, k, d), dtype=torch.float32, device="cuda")
        W = torch.zeros((d, d), dtype=torch.float32, device="cuda")
        with pytest.raises(SAError) as e:
            q.backward(dev["X"], dev["offsets"], G, P_f32=torch.zeros((k, d), device="cuda"),
                       W_Q_f32=W, W_K_f32=W)
        assert e.value.status == SA_ERR_UNSUPPORTED
        q.close()
