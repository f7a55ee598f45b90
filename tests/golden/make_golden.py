"""Writes tests/golden/tiny_oracle.json: the oracle's routing and a slice of
its output on the tiny workload (T=16, d=256, E=16, k=2, f=64).

Calls only oracle/ and the seeded input generator.  Re-run it only with a
commit message that names the passage (or its reading) that justifies a
change of the oracle's arithmetic.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_diffusion_moe_router_b200 import inputs  # noqa: E402


def main():
    w = inputs.WORKLOADS["tiny"]
    lay = inputs.make_layer(w)
    out, idx, wts, gap = oracle.moe_forward(lay["x"], lay["router_w"], lay["router_gamma"],
                                            None, lay["w_gate_up"], lay["w_down"], w.k)
    doc = {
        "workload": "tiny T=16 d=256 E=16 k=2 f=64 bf16, seeds 0..9, eps 1e-6",
        "idx": idx.tolist(),
        "w": [[float(v) for v in row] for row in wts],
        "gap": [float(v) for v in gap],
        "out_rows_0_1_cols_0_16": [[float(v) for v in out[t, :16]] for t in range(2)],
        "out_l2": float((out ** 2).sum() ** 0.5),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as fh:
        json.dump(doc, fh, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
