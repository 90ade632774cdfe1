"""Writes ``oracle_small_cases.json``: small seeded SA cases and the oracle's
outputs for them, frozen so that any later change to the oracle's arithmetic
shows up as a test failure (and must then be justified by a passage of the
SequenceO1 reading notes in its commit message).

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

from oracle import sa_batch  # noqa: E402
from synthetic.workloads import make_inputs  # noqa: E402

CASES = [
    dict(name="three_users_one_empty", lengths=[3, 0, 5], d=4, k=3, dtype="fp32", seed=5),
    dict(name="bf16_inputs", lengths=[7, 2], d=8, k=4, dtype="bf16", seed=6),
    dict(name="single_row_user", lengths=[1], d=4, k=5, dtype="fp32", seed=8),
]


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


if __name__ == "__main__":
    main()
