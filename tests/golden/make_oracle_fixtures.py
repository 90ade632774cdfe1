"""Writes ``oracle_small_cases.json`` (small seeded SA cases and the oracle's
outputs for them) and ``oracle_refinement_cases.json`` (per-user queries,
section 2.2, and the gradients of a layer), frozen so that any later change
to the oracle's arithmetic shows up as a test failure (and must then be
justified by a passage of the SequenceO1 reading notes in its commit
message).

The pages print no worked numerical example of an SA layer, so no fixture
here holds values taken from them; the pinned facts live in
``tests/oracle_pins.py``.

This script calls only ``oracle/`` and ``synthetic/``.  Run from the repo
root:  python tests/golden/make_oracle_fixtures.py
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import sa_batch, sa_batch_backward, sa_batch_user_queries  # noqa: E402
from synthetic.workloads import make_inputs, upstream_gradients, user_queries  # noqa: E402

CASES = [
    dict(name="three_users_one_empty", lengths=[3, 0, 5], d=4, k=3, dtype="fp32", seed=5),
    dict(name="bf16_inputs", lengths=[7, 2], d=8, k=4, dtype="bf16", seed=6),
    dict(name="single_row_user", lengths=[1], d=4, k=5, dtype="fp32", seed=8),
]


REFINEMENT_CASES = [
    dict(name="user_queries_ragged", kind="user_queries", lengths=[3, 0, 5], d=4, k=3,
         dtype="fp32", seed=15),
    dict(name="backward_shared_prototypes", kind="backward", lengths=[4, 0, 3], d=4, k=3,
         dtype="fp32", seed=16),
    dict(name="backward_user_queries", kind="backward_user_queries", lengths=[2, 5], d=4, k=2,
         dtype="bf16", seed=17),
]


def refinement_entry(c):
    inp = make_inputs(c["lengths"], c["d"], c["k"], c["dtype"], c["seed"])
    B = len(c["lengths"])
    out = dict(case=c)
    if c["kind"] == "user_queries":
        Q = user_queries(B, c["k"], c["d"], seed=c["seed"])
        Xt, m = sa_batch_user_queries(inp["X"], inp["offsets"], Q, inp["W_Q"], inp["W_K"],
                                      inp["scale"])
        out.update(X_tilde=Xt.tolist(), mass=m.tolist())
    else:
        G, g = upstream_gradients(B, c["k"], c["d"], seed=c["seed"])
        Q = user_queries(B, c["k"], c["d"], seed=c["seed"]) \
            if c["kind"] == "backward_user_queries" else None
        r = sa_batch_backward(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                              inp["scale"], G, g, queries=Q)
        out.update({key: val.tolist() for key, val in r.items()})
    return out


def main():
    out = []
    for c in CASES:
        inp = make_inputs(c["lengths"], c["d"], c["k"], c["dtype"], c["seed"])
        Xt, m = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"],
                         inp["scale"])
        out.append(dict(case=c, X_tilde=Xt.tolist(), mass=m.tolist()))
    with open(os.path.join(HERE, "oracle_small_cases.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    with open(os.path.join(HERE, "oracle_refinement_cases.json"), "w") as f:
        json.dump([refinement_entry(c) for c in REFINEMENT_CASES], f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
