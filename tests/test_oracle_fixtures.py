"""The oracle still reproduces its frozen small cases (regression guard),
for the SA layer, per-user queries and the layer's gradients."""

import json
import os

import numpy as np
import pytest

import sys

from oracle import sa_batch
from synthetic.workloads import make_inputs

sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
from make_oracle_fixtures import refinement_entry  # noqa: E402

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


REF_PATH = os.path.join(os.path.dirname(__file__), "golden", "oracle_refinement_cases.json")
with open(REF_PATH) as f:
    REF_CASES = json.load(f)


@pytest.mark.parametrize("entry", REF_CASES, ids=lambda e: e["case"]["name"])
def test_oracle_matches_frozen_refinement_case(entry):
    now = refinement_entry(entry["case"])
    keys = [key for key in entry if key != "case"]
    assert sorted(keys) == sorted(key for key in now if key != "case")
    for key in keys:
        np.testing.assert_allclose(np.array(now[key]), np.array(entry[key]), rtol=1e-13,
                                   atol=1e-15, err_msg=key)
