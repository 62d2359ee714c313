"""Writes tiny_oracle.json: the fp64 oracle's output on the tiny workload
(batch 1, 8x8 grid, 1 head, d_k = d_v = 16, mild gates, seed 0) for the L->R
and T->B scan orders.  Calls only the oracle and the seeded input generator;
nothing here comes from the CUDA path.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle  # noqa: E402
from recurrent_vision_backbone_key_b200.synthetic import make_inputs  # noqa: E402

W = dict(B=1, grid_h=8, grid_w=8, heads=1, d_k=16, d_v=16, seed=0, gate="mild")


def main():
    q, k, v, g = make_inputs(W["B"], W["grid_h"], W["grid_w"], W["heads"], W["d_k"], W["d_v"],
                             seed=W["seed"], gate=W["gate"])
    doc = {"workload": W,
           "source": "fp64 oracle (oracle/gla_oracle.c), serial recurrence",
           "layout": "[B, N, heads, d_v] flattened, row-major spatial token order"}
    for key, direction in (("l2r", 0), ("t2b", 2)):
        out = oracle.gla_serial(q, k, v, g, W["grid_h"], W["grid_w"], direction)
        doc[key] = [float(x) for x in out.reshape(-1)]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
