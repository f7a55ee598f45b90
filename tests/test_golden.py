"""Golden fixtures: the constants the pages fix, and the oracle's frozen
output on the tiny workload (written by tests/golden/make_golden.py)."""
import json
import os

import numpy as np

import oracle
from block_diffusion_moe_router_b200 import inputs

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_workloads_use_page_constants():
    c = json.load(open(os.path.join(HERE, "page_constants.json")))
    for name in ("canvas", "canvas4", "encode", "stack30"):
        w = inputs.WORKLOADS[name]
        assert w.E == c["n_experts"]["value"]
        assert w.k == c["top_k"]["value"]
        assert w.d == c["hidden"]["value"]
        assert w.f == c["expert_intermediate"]["value"]
    assert inputs.WORKLOADS["canvas"].T == c["canvas_tokens"]["value"]
    assert inputs.WORKLOADS["encode"].T == c["prompt_plus_canvas_ctx"]["value"]
    assert inputs.WORKLOADS["stack30"].layers == c["moe_layers_per_stack"]["value"]
    assert 2 * inputs.WORKLOADS["stack30"].layers == c["moe_modules"]["value"]
    assert inputs.GROUP == c["int4_group_size"]["value"]


def test_oracle_reproduces_frozen_tiny_output():
    g = json.load(open(os.path.join(HERE, "tiny_oracle.json")))
    w = inputs.WORKLOADS["tiny"]
    lay = inputs.make_layer(w)
    out, idx, wts, gap = oracle.moe_forward(lay["x"], lay["router_w"], lay["router_gamma"],
                                            None, lay["w_gate_up"], lay["w_down"], w.k)
    assert idx.tolist() == g["idx"]
    np.testing.assert_allclose(wts, np.array(g["w"]), rtol=1e-12)
    np.testing.assert_allclose(gap, np.array(g["gap"]), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(out[:2, :16], np.array(g["out_rows_0_1_cols_0_16"]), rtol=1e-12)
    assert abs(float((out ** 2).sum() ** 0.5) - g["out_l2"]) < 1e-9 * g["out_l2"]
