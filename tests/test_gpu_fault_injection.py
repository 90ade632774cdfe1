"""Failure detection without a GPU fault: the fault-injection build
(libsa_inject.so: the same sources with a 2e8-cycle wait limit and a device
switch) makes CTA 0 of the fused pass skip one X copy, so MMA1 waits on a
barrier that nothing completes.  The wait runs out, every role stops, the
copies and MMAs in flight finish, the tensor memory is released, and the host
reads DEVFLAG_TIMEOUT.  The same context then runs a clean layer that matches
the oracle.  The product library (libsa.so) has no such switch."""

import ctypes
import os
import time

import numpy as np
import pytest

from gpu_util import assert_user_close, to_device
from oracle import sa_batch
from synthetic.workloads import make_inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INJECT_LIB = os.path.join(ROOT, "sketch_attention_compression_b200", "_lib", "libsa_inject.so")


def _run(binding, dev, inp):
    q = binding.SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    B = len(inp["offsets"]) - 1
    ws = q.new_workspace(B, dev["X"].shape[0])
    Xt, m = q.forward(dev["X"], dev["offsets"], workspace=ws)
    flags = binding.read_device_status(ws)
    out = (Xt.double().cpu().numpy(), m.double().cpu().numpy(), flags)
    q.close()
    return out


def test_stalled_copy_reports_timeout_and_context_survives():
    import torch

    from sketch_attention_compression_b200 import binding

    assert os.path.exists(INJECT_LIB), "build libsa_inject.so first (build.build_all())"
    inp = make_inputs([400_000], d=128, k=128, dtype="bf16", seed=31)
    dev = to_device(inp)
    product = binding.load_library()
    assert not hasattr(product, "sa_debug_inject_stall")
    saved = binding._lib
    lib = binding.load_library(INJECT_LIB)
    lib.sa_debug_inject_stall.restype = ctypes.c_int
    lib.sa_debug_inject_stall.argtypes = [ctypes.c_int]
    binding._lib = lib
    try:
        assert lib.sa_debug_inject_stall(5) == 0
        t0 = time.time()
        _, _, flags = _run(binding, dev, inp)
        torch.cuda.synchronize()
        elapsed = time.time() - t0
        assert flags & binding.DEVFLAG_TIMEOUT, f"flags {flags}"
        assert elapsed < 30, f"the stalled call took {elapsed:.1f} s"

        assert lib.sa_debug_inject_stall(-1) == 0
        Xt, m, flags = _run(binding, dev, inp)
        assert flags == 0
        Xo, mo = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
        assert_user_close(Xt[0], m[0], Xo[0], mo[0], "bf16", "after the stalled call")
    finally:
        lib.sa_debug_inject_stall(-1)
        binding._lib = saved
    # and the product library still works on this context
    Xt, m, flags = _run(binding, dev, inp)
    assert flags == 0
