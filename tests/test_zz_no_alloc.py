"""sa_sketch_forward_noalloc: the entry point for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc where they run the SA
layer: code inside an allocator's own hooks, code under a memory pool that
must not grow, hosts that hand over only fixed buffers.  For them the library
keeps a fixed scratch array in its device image instead of asking for a
workspace.  These tests call that entry point through the C ABI and check it
against the CPU oracle and against sa_sketch_forward (the workspace path) on
two calls in a row with different inputs, so that the second call runs on
scratch the first one left behind; that the device flags it reports belong
to the call that raised them; and that, once set up, a call takes no device
memory.

The file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.  Each test also passes when
run alone in a fresh process (the first call on the device does the set-up).
"""

import numpy as np
import pytest

from gpu_util import TOL, assert_total_mass, assert_user_close, to_device
from oracle import sa_batch
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu

SA_DEVFLAG_OFFSET_LAST = 4


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
    _close(Xt_n, Xt_w, inp["dtype"], "X~ vs workspace path")
    _close(m_n, m_w, inp["dtype"], "m vs workspace path")
    Xt_o, m_o = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                         inp["scale"])
    Xg, mg = Xt_n.double().cpu().numpy(), m_n.double().cpu().numpy()
    for b in range(len(inp["offsets"]) - 1):
        assert_user_close(Xg[b], mg[b], Xt_o[b], m_o[b], inp["dtype"], f"oracle user {b}")
    assert_total_mass(mg, inp["offsets"], inp["dtype"])
    q.close()


def test_noalloc_matches_oracle_and_workspace_path_two_calls():
    # Call 1: users that cross CTA row ranges, so partial slots are used.
    _one_call(make_inputs([70_000, 129, 30_000, 0, 1], d=128, k=128, dtype="bf16", seed=41))
    # Call 2: other shapes on the scratch call 1 left behind.
    _one_call(make_inputs([5_000, 0, 40_000, 127, 3], d=64, k=33, dtype="bf16", seed=42))


def test_noalloc_flags_belong_to_their_call():
    """A call with offsets[B] != N reports SA_DEVFLAG_OFFSET_LAST; the clean
    call after it on the same scratch reports nothing; a batch = 0 call (the
    set-up call) writes zeros over whatever the flag words held."""
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    inp = make_inputs([3000, 500], d=128, k=64, dtype="bf16", seed=44)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    flags = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    bad = torch.tensor([0, 3000, 3499], dtype=torch.int64, device="cuda")  # N is 3500
    q.forward_noalloc(dev["X"], bad, device_flags=flags)
    torch.cuda.synchronize()
    assert flags[0].item() & SA_DEVFLAG_OFFSET_LAST
    assert flags[1].item() == 0
    flags.fill_(-1)
    q.forward_noalloc(dev["X"], dev["offsets"], device_flags=flags)
    torch.cuda.synchronize()
    assert flags.tolist() == [0, 0]
    flags.fill_(-1)
    X0 = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    off0 = torch.zeros(1, dtype=torch.int64, device="cuda")
    Xt0 = torch.empty((1, 64, 128), dtype=torch.float32, device="cuda")
    m0 = torch.empty((1, 64), dtype=torch.float32, device="cuda")
    q.forward_noalloc(X0, off0, Xt0[:0], m0[:0], device_flags=flags)
    torch.cuda.synchronize()
    assert flags.tolist() == [0, 0]
    q.close()


def test_noalloc_takes_no_device_memory_after_set_up():
    """After the first call on the device (the set-up), a call leaves the
    device's free memory unchanged: it allocates nothing."""
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    inp = make_inputs([60_000, 7, 20_000], d=128, k=128, dtype="bf16", seed=45)
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    B = len(inp["offsets"]) - 1
    Xt = torch.empty((B, 128, 128), dtype=torch.float32, device="cuda")
    m = torch.empty((B, 128), dtype=torch.float32, device="cuda")
    flags = torch.zeros(2, dtype=torch.int32, device="cuda")
    q.forward_noalloc(dev["X"], dev["offsets"], Xt, m, device_flags=flags)  # set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        q.forward_noalloc(dev["X"], dev["offsets"], Xt, m, device_flags=flags)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory moved by {free0 - free1} bytes"
    assert flags.tolist() == [0, 0]
    q.close()


def test_noalloc_rejects_queries_beyond_the_scratch():
    from sketch_attention_compression_b200 import SAError, SketchQuery
    from sketch_attention_compression_b200.binding import SA_ERR_WORKSPACE
    inp = make_inputs([20_000], d=256, k=256, dtype="fp32", seed=43)  # 148 CTA ranges
    dev = to_device(inp)
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    with pytest.raises(SAError) as e:
        q.forward_noalloc(dev["X"], dev["offsets"])
    assert e.value.status == SA_ERR_WORKSPACE
    q.close()
