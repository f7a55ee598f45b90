"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle
on the same seeded inputs, element by element."""
import numpy as np
import pytest
import torch

import oracle
from block_diffusion_moe_router_b200 import inputs
import block_diffusion_moe_router_b200 as moe
from parity_util import (TOL_BF16, check_routing, oracle_rows_for_sets, rel_l2, stable_tables)

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _cuda(lay):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}


def _cpu(lay):
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}


def run_gpu(layer, lay_gpu, T, residual=None, out=None):
    x = lay_gpu["x"]
    out = layer.forward(x, lay_gpu["router_w"], lay_gpu["router_gamma"], lay_gpu["w_gate_up"],
                        lay_gpu["w_down"], router_bias=lay_gpu.get("router_bias"),
                        scales_gate_up=lay_gpu.get("scales_gate_up"),
                        scales_down=lay_gpu.get("scales_down"), residual=residual, out=out)
    st = layer.sync_status()
    assert st == moe.MOE_OK, moe.moe_status_str(st)
    return out


def full_check(lay_cpu, lay_gpu, E, k, d, f, rows=None, residual=None, tol=TOL_BF16,
               check_tables=True):
    """Runs route + forward on the GPU and compares with the oracle (all rows
    or the sampled `rows`)."""
    T = lay_gpu["x"].shape[0]
    layer = moe.MoeLayer(E, k, d, f, lay_gpu.get("wdtype", moe.MOE_W_BF16))
    try:
        gidx, gw, ggap = layer.route(lay_gpu["x"], lay_gpu["router_w"], lay_gpu["router_gamma"],
                                     lay_gpu.get("router_bias"))
        out = run_gpu(layer, lay_gpu, T, residual=residual)
        torch.cuda.synchronize()
        tables = [t.cpu().numpy() for t in layer.routing_tables(T)] if check_tables else None
    finally:
        layer.close()
    sel = np.arange(T) if rows is None else np.asarray(rows)
    sub = dict(lay_cpu)
    sub["x"] = lay_cpu["x"][sel]
    res_cpu = residual.cpu()[sel] if residual is not None else None
    ref, oidx, ow, ogap = oracle.moe_forward(sub["x"], sub["router_w"], sub["router_gamma"],
                                             sub.get("router_bias"), sub["w_gate_up"],
                                             sub["w_down"], k,
                                             scales_gate_up=sub.get("scales_gate_up"),
                                             scales_down=sub.get("scales_down"),
                                             residual=res_cpu, eps=EPS)
    _, _, _, z = oracle.route(sub["x"], sub["router_w"], sub["router_gamma"],
                              sub.get("router_bias"), k, eps=EPS)
    gidx_s = gidx.cpu().numpy()[sel]
    mism = check_routing(gidx_s, gw.cpu().numpy()[sel], oidx, ow, ogap, z, k)
    got = out.float().cpu().numpy()[sel].astype(np.float64)
    if len(mism):
        sub2 = dict(sub)
        if res_cpu is not None:
            sub2["residual"] = res_cpu
        ref = ref.copy()
        ref[mism] = oracle_rows_for_sets(sub2, k, mism, [set(gidx_s[t]) for t in mism], eps=EPS)
    err = rel_l2(got, ref)
    assert err <= tol, f"rel-L2 {err:.3e} > {tol}"
    # gap reported by the router kernel (+inf when k == E)
    gg = ggap.cpu().numpy()[sel]
    fin = np.isfinite(ogap)
    assert np.all(np.isinf(gg[~fin]))
    np.testing.assert_allclose(gg[fin], ogap[fin], rtol=1e-3, atol=2e-5)
    # routing tables bit-exact (when the sets agree everywhere)
    if check_tables and rows is None and len(mism) == 0:
        off, perm, slot_of = stable_tables(oidx, E)
        assert np.array_equal(tables[0], off)
        assert np.array_equal(tables[1], perm)
        assert np.array_equal(tables[2], slot_of)
    return err, out


# ------------------------------------------------------------------ configs


@pytest.fixture(scope="module")
def canvas():
    w = inputs.WORKLOADS["canvas"]
    lay_gpu = inputs.make_layer(w, device="cuda")
    return w, _cpu(lay_gpu), lay_gpu


def test_tiny_workload():
    w = inputs.WORKLOADS["tiny"]
    lay = inputs.make_layer(w)
    err, _ = full_check(lay, _cuda(lay), w.E, w.k, w.d, w.f)
    print("tiny rel-L2", err)


def test_canvas_full_layer(canvas):
    """T=256, d=2816, E=128, k=8, f=704, bf16: every token against the oracle."""
    w, lay_cpu, lay_gpu = canvas
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f)
    print("canvas rel-L2", err)


def test_canvas_deterministic(canvas):
    w, lay_cpu, lay_gpu = canvas
    layer = moe.MoeLayer(w.E, w.k, w.d, w.f)
    try:
        a = run_gpu(layer, lay_gpu, w.T).clone()
        b = run_gpu(layer, lay_gpu, w.T).clone()
    finally:
        layer.close()
    assert torch.equal(a, b)


def test_encode_sampled_rows():
    """T=2048 (prompt + canvas): the GPU runs every token; the oracle checks a
    seeded sample of 160 rows including the first and last tiles."""
    w = inputs.WORKLOADS["encode"]
    lay_gpu = inputs.make_layer(w, device="cuda")
    lay_cpu = _cpu(lay_gpu)
    g = np.random.default_rng(3)
    rows = np.unique(np.concatenate([np.arange(16), np.arange(w.T - 16, w.T),
                                     g.choice(w.T, 128, replace=False)]))
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f, rows=rows)
    print("encode sampled rel-L2", err)


def test_stack30_layer_zipf_bias_and_residual():
    """One layer of the 30-layer stack: Zipf-skewed router bias, residual added
    in place (out aliases residual).  The delta is checked with the residual
    off, the residual path on the full output."""
    w = inputs.WORKLOADS["stack30"]
    lay_gpu = inputs.make_layer(w, layer=7, device="cuda")
    lay_cpu = _cpu(lay_gpu)
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f)
    res = inputs._randn((w.T, w.d), 1.0, 4242, "cuda", torch.bfloat16)
    layer = moe.MoeLayer(w.E, w.k, w.d, w.f)
    try:
        delta = run_gpu(layer, lay_gpu, w.T).float()
        buf = res.clone()
        out = run_gpu(layer, lay_gpu, w.T, residual=buf, out=buf).float()
    finally:
        layer.close()
    want = (res.float() + delta).to(torch.bfloat16).float()
    # out = bf16(residual + delta) with delta unrounded; `want` used the bf16
    # delta: they differ by at most one bf16 ulp of out plus delta's rounding
    bound = want.abs() * 2.0 ** -7 + delta.abs() * 2.0 ** -8 + 1e-6
    assert torch.all((out - want).abs() <= bound)
    print("stack30 layer delta rel-L2", err)


# ------------------------------------------------------------------ edge cases


@pytest.mark.parametrize("T,E,k,d,f,bias", [
    (1, 16, 2, 256, 64, False),      # single token
    (17, 16, 2, 256, 64, True),      # ragged router tile / tails
    (40, 8, 8, 256, 128, False),     # E == k: every expert used
    (9, 1, 1, 128, 64, False),       # dense gated FFN
    (300, 33, 3, 384, 192, True),    # E not a multiple of 32, f not of 128
])
def test_edge_shapes(T, E, k, d, f, bias):
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=T + E, bias=bias)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f)
    print((T, E, k, d, f), "rel-L2", err)


def test_hot_expert_multi_chunk():
    """One expert receives every token (T=600 > 256): its work splits into
    three 256-token chunks; the widest B stage is exercised."""
    T, E, k, d, f = 600, 16, 2, 256, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=77, bias=True)
    lay["router_bias"] = torch.zeros(E)
    lay["router_bias"][5] = 50.0
    err, _ = full_check(lay, _cuda(lay), E, k, d, f)
    print("hot expert rel-L2", err)


def test_zero_tokens_is_noop():
    layer = moe.MoeLayer(16, 2, 256, 64)
    try:
        st = moe.moe_forward(layer.plan, 0, None, None, None, None, None, None, None, None, None,
                             None, check=False)
        assert st == moe.MOE_OK
    finally:
        layer.close()


def test_forward_host_matches_device(canvas):
    w, lay_cpu, lay_gpu = canvas
    layer = moe.MoeLayer(w.E, w.k, w.d, w.f)
    try:
        dev_out = run_gpu(layer, lay_gpu, w.T).cpu()
        x_h = lay_cpu["x"].pin_memory()
        out_h = torch.empty_like(x_h).pin_memory()
        moe.moe_forward_host(layer.plan, w.T, x_h, lay_gpu["router_w"], lay_gpu["router_gamma"],
                             None, lay_gpu["w_gate_up"], lay_gpu["w_down"], None, None, None,
                             out_h)
        assert layer.sync_status() == moe.MOE_OK
    finally:
        layer.close()
    assert torch.equal(out_h, dev_out)


# ------------------------------------------------------------------ error paths


def test_invalid_arguments_launch_nothing():
    T, E, k, d, f = 8, 16, 2, 256, 64
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=1))
    layer = moe.MoeLayer(E, k, d, f)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    args = [lay["x"], lay["router_w"], lay["router_gamma"], None, lay["w_gate_up"],
            lay["w_down"], None, None, None, out]

    def call(*a, T_=T):
        return moe.moe_forward(layer.plan, T_, *a, check=False)

    try:
        assert call(*args) == moe.MOE_OK
        assert call(*args, T_=-1) == moe.MOE_ERR_INVALID_ARG
        bad = list(args)
        bad[0] = None
        assert call(*bad) == moe.MOE_ERR_INVALID_ARG
        bad = list(args)
        bad[0] = lay["x"].data_ptr() + 2  # misaligned
        assert call(*bad) == moe.MOE_ERR_INVALID_ARG
        bad = list(args)
        bad[9] = lay["x"]  # out overlaps x
        assert call(*bad) == moe.MOE_ERR_INVALID_ARG
        bad = list(args)
        bad[6] = lay["w_gate_up"]  # scales given to a bf16 plan
        assert call(*bad) == moe.MOE_ERR_INVALID_ARG
        assert layer.sync_status() == moe.MOE_OK
    finally:
        layer.close()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_plan_create(16, 17, 256, 64)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED


def test_bounded_wait_reports_timeout_and_context_survives():
    """The expert kernel's dependency wait is pointed at a flag nothing sets:
    the bounded wait runs out, the call reports MOE_ERR_TIMEOUT, and the next
    call on the same context is correct."""
    T, E, k, d, f = 32, 16, 2, 256, 64
    lay_cpu = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=2)
    lay = _cuda(lay_cpu)
    layer = moe.MoeLayer(E, k, d, f)
    try:
        good = run_gpu(layer, lay, T).clone()
        moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_TIMEOUT_MS, 20)
        moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_TEST_STALL, 1)
        layer.forward(lay["x"], lay["router_w"], lay["router_gamma"], lay["w_gate_up"],
                      lay["w_down"])
        assert layer.sync_status() == moe.MOE_ERR_TIMEOUT
        moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_TEST_STALL, 0)
        again = run_gpu(layer, lay, T)
        assert torch.equal(again, good)
    finally:
        layer.close()
