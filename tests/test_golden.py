"""The oracle against its own stored output (tests/golden/oracle_c1_rows.json, written
by tests/golden/make_golden.py, which calls only oracle/): a change to the oracle's
arithmetic shows up here as a difference."""
import json
import os

import numpy as np

import oracle
from workloads import WORKLOADS, make_inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_stored_rows():
    with open(os.path.join(HERE, "golden", "oracle_c1_rows.json")) as f:
        g = json.load(f)
    w = WORKLOADS[g["workload"]]
    q, k, v = (t.double().numpy() for t in make_inputs(w))
    for name, case in g["cases"].items():
        o, lse = oracle.attn_ref(q, k, v, name == "causal", g["scale"])
        for r, (b, h, i) in enumerate(g["rows"]):
            np.testing.assert_allclose(o[b, h, i], case["o"][r], rtol=1e-14, atol=1e-15)
            np.testing.assert_allclose(lse[b, h, i], case["lse"][r], rtol=1e-14, atol=1e-15)
