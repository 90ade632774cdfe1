"""Helpers for the GPU parity tests: move seeded inputs to the device, run
the CUDA path through the C ABI, compare with the oracle."""

from __future__ import annotations

import numpy as np

# Tolerances: max |X~_gpu - X~_oracle| <= TOL * max |X~_oracle| per user
# (same rule for the mass); bf16 inputs with fp32 accumulation: 2e-2; fp32
# path: 1e-4.
# |sum_j m_j - n_b| <= MASS_SUM_TOL * n_b: on the bf16 path each row's
# probabilities (which sum to 1 in fp32) are rounded to bf16, relative error
# at most 2^-8 each, and the masses are sums of those same rounded values,
# so a row adds at most 2^-8 to the deviation; the fp32 path keeps fp32
# probabilities and fp64 sums.
TOL = {"bf16": 2e-2, "fp32": 1e-4}
MASS_SUM_TOL = {"bf16": 2.0 ** -8, "fp32": 1e-5}


def torch_dtype(dtype: str):
    import torch
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_device(inp: dict) -> dict:
    import torch
    dt = torch_dtype(inp["dtype"])
    dev = torch.device("cuda")
    out = {key: torch.from_numpy(np.ascontiguousarray(inp[key])).to(dev).to(dt)
           for key in ("X", "P", "W_Q", "W_K")}
    out["offsets"] = torch.from_numpy(np.ascontiguousarray(inp["offsets"])).to(dev)
    return out


def run_gpu(inp: dict, dev: dict | None = None, check: bool = True):
    """Returns (X~ (B,k,d), m (B,k)) as float64 numpy arrays and the device flags."""
    import torch
    from sketch_attention_compression_b200 import SketchQuery, read_device_status
    dev = to_device(inp) if dev is None else dev
    q = SketchQuery(dev["P"], dev["W_Q"], dev["W_K"], inp["scale"])
    B = len(inp["offsets"]) - 1
    ws = q.new_workspace(B, dev["X"].shape[0])
    Xt, m = q.forward(dev["X"], dev["offsets"], workspace=ws)
    flags = read_device_status(ws) if check else 0
    torch.cuda.synchronize()
    out = (Xt.double().cpu().numpy(), m.double().cpu().numpy(), flags)
    q.close()
    return out


def assert_user_close(Xt_g, m_g, Xt_o, m_o, dtype, what=""):
    tol = TOL[dtype]
    ref_x = max(np.max(np.abs(Xt_o)), 1e-30)
    err_x = np.max(np.abs(Xt_g - Xt_o))
    ref_m = max(np.max(np.abs(m_o)), 1e-30)
    err_m = np.max(np.abs(m_g - m_o))
    assert np.all(np.isfinite(Xt_g)) and np.all(np.isfinite(m_g)), f"{what}: non-finite"
    assert err_x <= tol * ref_x, f"{what}: X~ err {err_x:.3e} > {tol} * {ref_x:.3e}"
    assert err_m <= tol * ref_m, f"{what}: m err {err_m:.3e} > {tol} * {ref_m:.3e}"
    return err_x / ref_x, err_m / ref_m


def assert_total_mass(m_g, offsets, dtype):
    n = np.diff(np.asarray(offsets)).astype(np.float64)
    tot = m_g.sum(axis=1)
    bad = np.abs(tot - n) > MASS_SUM_TOL[dtype] * np.maximum(n, 1.0)
    assert not bad.any(), f"sum_j m_j != n_b for users {np.nonzero(bad)[0][:10]}"
