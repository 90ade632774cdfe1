"""The oracle still reproduces its frozen small cases (regression guard)."""

import json
import os

import numpy as np
import pytest

from oracle import sa_batch
from synthetic.workloads import make_inputs

PATH = os.path.join(os.path.dirname(__file__), "golden", "oracle_small_cases.json")
with open(PATH) as f:
    CASES = json.load(f)


@pytest.mark.parametrize("entry", CASES, ids=lambda e: e["case"]["name"])
def test_oracle_matches_frozen_case(entry):
    c = entry["case"]
    inp = make_inputs(c["lengths"], c["d"], c["k"], c["dtype"], c["seed"])
    Xt, m = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                     inp["scale"])
    np.testing.assert_allclose(Xt, np.array(entry["X_tilde"]), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(m, np.array(entry["mass"]), rtol=1e-13, atol=1e-15)
