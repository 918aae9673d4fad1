"""Write oracle_c1_rows.json: sampled rows of the fp64 oracle's output on the tiny
seeded workload (B=1, H=2, Sq=Sk=128, D=64, fp16 inputs from seed 0, scale 1/8), both
causal modes.  Calls only oracle/ and the shared input generator; run from the repo
root:  python tests/golden/make_golden.py"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import WORKLOADS, make_inputs  # noqa: E402

ROWS = [(0, 0, 0), (0, 0, 1), (0, 0, 63), (0, 1, 64), (0, 1, 126), (0, 1, 127)]


def compute():
    w = WORKLOADS["C1"]
    q, k, v = (t.double().numpy() for t in make_inputs(w))
    out = {"workload": "C1", "scale": w.scale, "rows": ROWS, "cases": {}}
    for causal in (False, True):
        o, lse = oracle.attn_ref(q, k, v, causal, w.scale)
        out["cases"]["causal" if causal else "noncausal"] = {
            "o": [[float(x) for x in o[b, h, i]] for (b, h, i) in ROWS],
            "lse": [float(lse[b, h, i]) for (b, h, i) in ROWS]}
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_c1_rows.json"), "w") as f:
        json.dump(compute(), f, indent=1)
        f.write("\n")
