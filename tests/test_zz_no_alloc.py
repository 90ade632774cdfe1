"""sa_sketch_forward_noalloc: the entry point for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc where they run the SA
layer (allocator hooks, pools that must not grow, hosts that hand over only
fixed buffers).  For them the library keeps a fixed scratch array in its
device image instead of asking for a workspace.  These tests call that entry
point through the C ABI and check it against sa_sketch_forward (the
workspace path) on two calls in a row with different inputs, so that the
second call runs on scratch the first one left behind.

The file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.
"""

import numpy as np
import pytest

from gpu_util import TOL, assert_total_mass, to_device
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu


def _close(a, b, dtype, what):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    for u in range(a.shape[0]):
        ref = max(np.abs(b[u]).max(), 1e-30)
        err = np.abs(a[u] - b[u]).max()
        assert err <= TOL[dtype] * ref, f"{what} user {u}: err {err:.3e} > {TOL[dtype]} * {ref:.3e}"


def _one_call(inp):
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    flags = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    Xt_n, m_n = q.forward_noalloc(dev["X"], dev["offsets"], device_flags=flags)
    Xt_w, m_w = q.forward(dev["X"], dev["offsets"])
    torch.cuda.synchronize()
    assert flags.tolist() == [0, 0]
    _close(Xt_n, Xt_w, inp["dtype"], "X~")
    _close(m_n, m_w, inp["dtype"], "m")
    assert_total_mass(m_n.double().cpu().numpy(), inp["offsets"], inp["dtype"])
    q.close()


def test_noalloc_matches_workspace_path_two_calls():
    # Call 1: users that cross CTA row ranges, so partial slots are used.
    _one_call(make_inputs([70_000, 129, 30_000, 0, 1], d=128, k=128, dtype="bf16", seed=41))
    # Call 2: other shapes on the scratch call 1 left behind.
    _one_call(make_inputs([5_000, 0, 40_000, 127, 3], d=64, k=33, dtype="bf16", seed=42))


def test_noalloc_rejects_queries_beyond_the_scratch():
    import torch
    from sketch_attention_compression_b200 import SAError, SketchQuery
    from sketch_attention_compression_b200.binding import SA_ERR_WORKSPACE
    inp = make_inputs([20_000], d=256, k=256, dtype="fp32", seed=43)  # 148 CTA ranges
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    with pytest.raises(SAError) as e:
        q.forward_noalloc(dev["X"], dev["offsets"])
    assert e.value.status == SA_ERR_WORKSPACE
    q.close()
