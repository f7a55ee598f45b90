"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle
on the same seeded inputs, element by element."""
import numpy as np
import pytest
import torch

import oracle
from block_diffusion_moe_router_b200 import inputs
import block_diffusion_moe_router_b200 as moe
from parity_util import (GAP_FLAG, TOL_BF16, TOL_FP4, TOL_FP8, TOL_INT4, check_routing,
                         oracle_rows_for_sets, rel_l2, stable_tables)

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
                        scales_down=lay_gpu.get("scales_down"), residual=residual, out=out,
                        expert_gamma=lay_gpu.get("expert_gamma"))
    st = layer.sync_status()
    assert st == moe.MOE_OK, moe.moe_status_str(st)
    return out


def full_check(lay_cpu, lay_gpu, E, k, d, f, rows=None, residual=None, tol=TOL_BF16,
               check_tables=True, options=None):
    """Runs route + forward on the GPU and compares with the oracle (all rows
    or the sampled `rows`); `options` are plan options set before the calls."""
    T = lay_gpu["x"].shape[0]
    coded = lay_gpu["w_gate_up"].dtype == torch.uint8
    fp8 = coded and lay_gpu["scales_gate_up"].dtype == torch.float32
    fp4 = coded and lay_gpu["scales_gate_up"].dtype == torch.uint8  # scale records
    int4 = coded and not fp8 and not fp4
    if int4 and tol == TOL_BF16:
        tol = TOL_INT4
    wdt = (moe.MOE_W_FP8_E4M3 if fp8 else moe.MOE_W_FP4_E2M1 if fp4
           else moe.MOE_W_INT4_G128 if int4 else moe.MOE_W_BF16)
    layer = moe.MoeLayer(E, k, d, f, wdt)
    try:
        for key, val in (options or {}).items():
            moe.moe_plan_set_option(layer.plan, key, val)
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
                                             residual=res_cpu, eps=EPS,
                                             expert_gamma=sub.get("expert_gamma"))
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


def test_canvas_y_fp32(canvas):
    """Expert outputs kept in fp32 before the combine (the default is bf16)."""
    w, lay_cpu, lay_gpu = canvas
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f, options={moe.MOE_OPT_Y_BF16: 0})
    print("canvas y-fp32 rel-L2", err)


@pytest.mark.parametrize("wd", [inputs.WDTYPE_BF16, inputs.WDTYPE_INT4, inputs.WDTYPE_FP8,
                                inputs.WDTYPE_FP4])
@pytest.mark.parametrize("ybf16", [0, 1])
def test_y_dtype_ragged_residual(wd, ybf16):
    """Both y precisions with a residual, ragged T and both weight formats."""
    lay = inputs.make_small(T=77, d=384, E=24, k=5, f=192, seed=61, wdtype=wd, bias=True,
                            residual=True)
    res = lay.pop("residual")
    err, _ = full_check(lay, _cuda(lay), 24, 5, 384, 192, residual=res.cuda(),
                        options={moe.MOE_OPT_Y_BF16: ybf16})
    print("ragged y-bf16" if ybf16 else "ragged y-fp32", "rel-L2", err)


@pytest.mark.parametrize("path", [1, 2])
def test_router_paths_canvas(canvas, path):
    """Both routers (tensor-core split-bf16 logits, FFMA fp32 logits) on the
    canvas: exact indices on unflagged tokens, weights and gaps close."""
    w, lay_cpu, lay_gpu = canvas
    layer = moe.MoeLayer(w.E, w.k, w.d, w.f)
    try:
        moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_ROUTER, path)
        gidx, gw, ggap = layer.route(lay_gpu["x"], lay_gpu["router_w"], lay_gpu["router_gamma"])
        assert layer.sync_status() == moe.MOE_OK
    finally:
        layer.close()
    oidx, ow, ogap, z = oracle.route(lay_cpu["x"], lay_cpu["router_w"], lay_cpu["router_gamma"],
                                     None, w.k, eps=EPS)
    check_routing(gidx.cpu().numpy(), gw.cpu().numpy(), oidx, ow, ogap, z, w.k)
    np.testing.assert_allclose(ggap.cpu().numpy(), ogap, rtol=1e-3, atol=2e-5)


def _triple_router(lay_cpu, E):
    """Router rows duplicated in triples: row e is a copy of row 3*(e//3)."""
    src = torch.arange(E) // 3 * 3
    return lay_cpu["router_w"][src].contiguous()


def _natural_near_ties(z, k, groups=4):
    """Tokens whose distinct logit values (ties between copies of one router
    row removed) come within the flag gap among the top `groups` values."""
    out = []
    for t in range(z.shape[0]):
        u = np.unique(z[t])[::-1][:groups + 1]
        if len(u) > 1 and np.min(u[:-1] - u[1:]) < 2 * GAP_FLAG:
            out.append(t)
    return set(out)


@pytest.mark.parametrize("path", [1, 2])
def test_exact_ties_lowest_index_both_routers(canvas, path):
    """Exact ties on the canvas: router rows duplicated in triples, so every
    token's logits come in equal threes and its top-8 takes whole triples
    (ties inside the selection, in index order) and then part of the next
    one (a tie across the 8th/9th boundary, broken toward the lower indices).
    Both routers must return the oracle's index arrays exactly, j order
    included, with no flag exemption for these ties; only tokens whose
    distinct logit values come within the flag gap of one another are exempt.
    Tied experts get bit-identical routing weights."""
    w, lay_cpu, lay_gpu = canvas
    rw = _triple_router(lay_cpu, w.E)
    layer = moe.MoeLayer(w.E, w.k, w.d, w.f)
    try:
        moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_ROUTER, path)
        gidx, gw, ggap = layer.route(lay_gpu["x"], rw.cuda(), lay_gpu["router_gamma"])
        assert layer.sync_status() == moe.MOE_OK
    finally:
        layer.close()
    oidx, ow, ogap, z = oracle.route(lay_cpu["x"], rw, lay_cpu["router_gamma"], None, w.k,
                                     eps=EPS)
    gidx, gw, ggap = gidx.cpu().numpy(), gw.cpu().numpy(), ggap.cpu().numpy()
    exempt = _natural_near_ties(z, w.k)
    assert len(exempt) <= 4, f"{len(exempt)} tokens with natural near-ties"
    check = np.array([t for t in range(w.T) if t not in exempt])
    # the construction puts an exact tie at the boundary on most tokens and
    # ties inside the selection on every token
    boundary_ties = int(np.sum(ogap[check] == 0.0))
    assert boundary_ties >= w.T // 2, boundary_ties
    np.testing.assert_array_equal(gidx[check], oidx[check])
    np.testing.assert_array_equal(ggap[check][ogap[check] == 0.0], 0.0)
    for t in check:
        for j in range(1, w.k):
            if z[t][oidx[t][j]] == z[t][oidx[t][j - 1]]:
                assert gw[t][j] == gw[t][j - 1], (t, j)
    np.testing.assert_allclose(gw[check], ow[check], rtol=1e-4, atol=1e-6)
    print(f"router path {path}: {boundary_ties} boundary ties, {len(exempt)} exempt tokens")


def test_exact_ties_full_layer(canvas):
    """The tie-laden router of the test above through the whole layer: the
    output matches the oracle (which takes the same lowest-index sets) and the
    routing tables are bit-exact."""
    w, lay_cpu, lay_gpu = canvas
    rw = _triple_router(lay_cpu, w.E)
    lc = dict(lay_cpu)
    lc["router_w"] = rw
    lg = dict(lay_gpu)
    lg["router_w"] = rw.cuda()
    err, _ = full_check(lc, lg, w.E, w.k, w.d, w.f)
    print("exact-tie canvas rel-L2", err)


def test_router_more_than_128_experts():
    """E = 200 (> 128) takes the FFMA router; top-8 still exact."""
    T, E, k, d, f = 40, 200, 8, 256, 64
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=200, bias=True)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f)
    print("E=200 rel-L2", err)


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


@pytest.mark.parametrize("wd", [inputs.WDTYPE_INT4, inputs.WDTYPE_FP8, inputs.WDTYPE_FP4])
def test_encode_shape_coded_weights_sampled_rows(wd):
    """T=2048 with int4, fp8 or fp4 expert weights: ~128 tokens per expert, so the
    coded kernels run their largest chunks (and the fp8 kernel its shallowest
    code ring); the oracle checks 48 sampled rows including both ends."""
    T, d, E, k, f = 2048, 2816, 128, 8, 704
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=120 + wd, wdtype=wd, device="cuda")
    lay_cpu = _cpu(lay)
    g = np.random.default_rng(4)
    rows = np.unique(np.concatenate([np.arange(8), np.arange(T - 8, T),
                                     g.choice(T, 32, replace=False)]))
    err, _ = full_check(lay_cpu, lay, E, k, d, f, rows=rows,
                        tol=TOL_INT4 if wd == inputs.WDTYPE_INT4 else TOL_FP8)
    print("encode-shape", {inputs.WDTYPE_INT4: "int4", inputs.WDTYPE_FP8: "fp8"}.get(wd, "fp4"),
          "sampled rel-L2", err)


@pytest.mark.parametrize("chunk", [0, 256])
def test_stack30_layer_zipf_bias_and_residual(chunk):
    """One layer of the 30-layer stack: Zipf-skewed router bias, residual added
    in place (out aliases residual).  The delta is checked with the residual
    off, the residual path on the full output.  chunk=0 cuts the hot experts'
    tokens into 128-token chunks (the default at one canvas), chunk=256 keeps
    each in one chunk of up to 256 tokens."""
    w = inputs.WORKLOADS["stack30"]
    lay_gpu = inputs.make_layer(w, layer=7, device="cuda")
    lay_cpu = _cpu(lay_gpu)
    opts = {moe.MOE_OPT_CHUNK_TOKENS: chunk}
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f, options=opts)
    res = inputs._randn((w.T, w.d), 1.0, 4242, "cuda", torch.bfloat16)
    layer = moe.MoeLayer(w.E, w.k, w.d, w.f)
    try:
        moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_CHUNK_TOKENS, chunk)
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


def test_canvas4_int4_full_layer():
    """T=256 canvas with symmetric int4 w4g128 expert weights (fp16 scales):
    every token against the oracle's exact code * scale arithmetic."""
    w = inputs.WORKLOADS["canvas4"]
    lay_gpu = inputs.make_layer(w, device="cuda")
    lay_cpu = _cpu(lay_gpu)
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f)
    print("canvas4 int4 rel-L2", err)


@pytest.mark.parametrize("T,E,k,d,f,bias", [
    (17, 16, 2, 256, 64, True),      # f=64: the only K stage of down is half out of bounds
    (300, 33, 3, 384, 192, False),   # f=192: last group of 64; E not a multiple of 32
])
def test_int4_edge_shapes(T, E, k, d, f, bias):
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=T + E + 1, bias=bias,
                            wdtype=inputs.WDTYPE_INT4)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f)
    print("int4", (T, E, k, d, f), "rel-L2", err)


def test_int4_hot_expert_chunks():
    """int4 units hold 128 tokens: one expert with 600 tokens spans 5 chunks."""
    T, E, k, d, f = 600, 16, 2, 256, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=78, bias=True,
                            wdtype=inputs.WDTYPE_INT4)
    lay["router_bias"] = torch.zeros(E)
    lay["router_bias"][3] = 50.0
    err, _ = full_check(lay, _cuda(lay), E, k, d, f)
    print("int4 hot expert rel-L2", err)


def test_canvas8_fp8_full_layer():
    """T=256 canvas with E4M3 expert weights and fp32 row scales: every
    token against the oracle's exact value * scale arithmetic."""
    w = inputs.WORKLOADS["canvas8"]
    lay_gpu = inputs.make_layer(w, device="cuda")
    lay_cpu = _cpu(lay_gpu)
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f, tol=TOL_FP8)
    print("canvas8 fp8 rel-L2", err)


@pytest.mark.parametrize("T,E,k,d,f,bias", [
    (17, 16, 2, 256, 64, True),      # f=64: the only K stage of down is half out of bounds
    (300, 33, 3, 384, 192, False),   # f=192: last stage of 64; E not a multiple of 32
    (1, 4, 1, 128, 128, False),      # one token, one 128-wide stage each way
])
def test_fp8_edge_shapes(T, E, k, d, f, bias):
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=T + E + 2, bias=bias,
                            wdtype=inputs.WDTYPE_FP8)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, tol=TOL_FP8)
    print("fp8", (T, E, k, d, f), "rel-L2", err)


def test_fp8_hot_expert_chunks():
    """fp8 units hold 128 tokens: one expert with 600 tokens spans 5 chunks."""
    T, E, k, d, f = 600, 16, 2, 256, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=79, bias=True,
                            wdtype=inputs.WDTYPE_FP8)
    lay["router_bias"] = torch.zeros(E)
    lay["router_bias"][3] = 50.0
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, tol=TOL_FP8)
    print("fp8 hot expert rel-L2", err)


@pytest.mark.parametrize("kind", ["subnormal", "extreme"])
def test_fp8_code_ranges(kind):
    """Every weight code subnormal (|v| < 2^-6), or every code at the
    format's largest magnitudes (+-256 .. +-448): the decode must be exact
    at both ends (a flushed subnormal or a saturated code would show)."""
    T, E, k, d, f = 33, 8, 2, 256, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=81, wdtype=inputs.WDTYPE_FP8)
    g = torch.Generator().manual_seed(5)
    for key in ("w_gate_up", "w_down"):
        shape = lay[key].shape
        sign = torch.randint(0, 2, shape, generator=g, dtype=torch.int32) << 7
        if kind == "subnormal":   # exponent 0, mantissa 1..7
            mag = torch.randint(1, 8, shape, generator=g, dtype=torch.int32)
        else:                     # exponent 15 (256 .. 448), mantissa 0..6
            mag = (15 << 3) | torch.randint(0, 7, shape, generator=g, dtype=torch.int32)
        lay[key] = (sign | mag).to(torch.uint8)
    # scales chosen so that the layer's values stay of order one
    amp = 2.0 ** 9 / 4 if kind == "subnormal" else 1.0 / 350
    lay["scales_gate_up"] = torch.full_like(lay["scales_gate_up"], amp * 0.02 * 3)
    lay["scales_down"] = torch.full_like(lay["scales_down"], amp * 0.02 * 3)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, tol=TOL_FP8)
    print("fp8", kind, "rel-L2", err)


def test_canvas4f_fp4_full_layer():
    """T=256 canvas with E2M1 expert weights, E4M3 scales per 16 weights and
    fp32 row scales: every token against the oracle's exact decode."""
    w = inputs.WORKLOADS["canvas4f"]
    lay_gpu = inputs.make_layer(w, device="cuda")
    lay_cpu = _cpu(lay_gpu)
    err, _ = full_check(lay_cpu, lay_gpu, w.E, w.k, w.d, w.f, tol=TOL_FP4)
    print("canvas4f fp4 rel-L2", err)


@pytest.mark.parametrize("T,E,k,d,f,bias", [
    (17, 16, 2, 256, 64, True),      # f=64: down's only K stage is half out of bounds (codes and blocks)
    (300, 33, 3, 384, 192, False),   # f=192: last stage of 64; E not a multiple of 32
    (1, 4, 1, 128, 128, False),      # one token, one 128-wide stage each way
])
def test_fp4_edge_shapes(T, E, k, d, f, bias):
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=T + E + 3, bias=bias,
                            wdtype=inputs.WDTYPE_FP4)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, tol=TOL_FP4)
    print("fp4", (T, E, k, d, f), "rel-L2", err)


def test_fp4_hot_expert_chunks():
    """fp4 units hold 128 tokens: one expert with 600 tokens spans 5 chunks."""
    T, E, k, d, f = 600, 16, 2, 256, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=83, bias=True,
                            wdtype=inputs.WDTYPE_FP4)
    lay["router_bias"] = torch.zeros(E)
    lay["router_bias"][3] = 50.0
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, tol=TOL_FP4)
    print("fp4 hot expert rel-L2", err)


@pytest.mark.parametrize("kind", ["subnormal", "extreme"])
def test_fp4_block_scale_ranges(kind):
    """Every E4M3 block scale subnormal (2^-9 .. 7 * 2^-9), or every one at
    the format's largest magnitudes (256 .. 448), over all 16 E2M1 codes: the
    scaled decode must stay exact at both ends (a flushed subnormal scale or an
    fp16 product out of range would show)."""
    T, E, k, d, f = 33, 8, 2, 256, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=85, wdtype=inputs.WDTYPE_FP4)
    g = torch.Generator().manual_seed(6)
    for key, (R, C) in (("scales_gate_up", (2 * f, d)), ("scales_down", (d, f))):
        rec = lay[key].clone()
        nb = C // inputs.FP4_BLOCK
        if kind == "subnormal":   # exponent 0, mantissa 1..7
            blk = torch.randint(1, 8, (E, nb * R), generator=g, dtype=torch.int32)
            srow = 2.0 ** 9 / 4 * 0.01
        else:                     # exponent 15, mantissa 0..6 (256 .. 448)
            blk = (15 << 3) | torch.randint(0, 7, (E, nb * R), generator=g, dtype=torch.int32)
            srow = 0.01 / 350
        rec[:, 4 * R:] = blk.to(torch.uint8)
        rows = torch.full((E, R), srow, dtype=torch.float32)
        rec[:, :4 * R] = rows.view(torch.uint8).reshape(E, 4 * R)
        lay[key] = rec
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, tol=TOL_FP4)
    print("fp4", kind, "rel-L2", err)


@pytest.mark.parametrize("wd", [inputs.WDTYPE_FP8, inputs.WDTYPE_FP4])
@pytest.mark.parametrize("T", [1, 16, 32, 33, 64, 65, 128, 129])
def test_coded_split_k_boundary(wd, T):
    """k = E: every expert gets all T tokens.  The fp8 and fp4 kernels split
    K between their two UMMA warps only for units of at most 64 tokens with
    two or more stage pairs: T=1 … 64 split (T=1 and 16 with UMMA N=16, 33
    across a 32-column step), 65 and 128 do not, 129 makes a 128-token chunk
    and a 1-token chunk that splits.  d=640 gives gate_up five K stages (a
    last pair of one stage), f=320 gives down three."""
    E = k = 2
    d, f = 640, 320
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=200 + T + wd, wdtype=wd)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, tol=TOL_FP8 if wd == inputs.WDTYPE_FP8 else TOL_FP4)
    print("split-K boundary", wd, T, "rel-L2", err)


@pytest.mark.parametrize("chunk", [0, 256])
@pytest.mark.parametrize("f", [64, 320])
@pytest.mark.parametrize("T", [1, 128, 129, 144, 145, 200, 256, 300])
def test_bf16_issuer_split_boundary(T, f, chunk):
    """k = E: every expert gets all T tokens.  The bf16 kernel's two UMMA
    issuers split K for a unit of at most 128 tokens with two or more K
    stages; a larger unit, or one of a single K stage, is one issuer's.
    d=640 gives gate_up ten K stages; f=320 gives down five, f=64 one (a
    single-issuer down unit at every T).  T=128/129 and 144/145 sit on either
    side of the split boundary and of a 16-column UMMA step; T=300 makes a
    256-token chunk next to a 44-token one, so the widest activation stage
    and a split unit share the ring.  With the default chunk size (chunk=0)
    a call of at most 256 tokens is cut into chunks of at most 128, so the
    single-issuer units above 128 tokens appear there only with chunk=256."""
    E = k = 2
    d = 640
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=400 + T + f)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f,
                        options={moe.MOE_OPT_CHUNK_TOKENS: chunk})
    print("issuer split boundary", T, f, chunk, "rel-L2", err)


# ------------------------------------------------------------------ edge cases


@pytest.mark.parametrize("T,E,k,d,f,bias", [
    (1, 16, 2, 256, 64, False),      # single token
    (17, 16, 2, 256, 64, True),      # ragged router tile / tails
    (40, 8, 8, 256, 128, False),     # E == k: every expert used
    (9, 1, 1, 128, 64, False),       # dense gated FFN
    (300, 33, 3, 384, 192, True),    # E not a multiple of 32, f not of 128
    (2200, 16, 8, 128, 64, False),   # > 16K assignments: a 9-CTA plan cluster
    (2048, 128, 8, 128, 64, False),  # the encode routing shape: an 8-CTA plan cluster
    (5000, 64, 8, 128, 64, True),    # 40K assignments: the 16-CTA plan cluster
])
def test_edge_shapes(T, E, k, d, f, bias):
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=T + E, bias=bias)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f)
    print((T, E, k, d, f), "rel-L2", err)


@pytest.mark.parametrize("wd", [inputs.WDTYPE_BF16, inputs.WDTYPE_INT4, inputs.WDTYPE_FP8,
                                inputs.WDTYPE_FP4])
def test_expert_side_norm(wd):
    """Experts read the (1+gamma2) RMSNorm of x (applied while gathering the
    rows); router and residual see the raw x."""
    T, E, k, d, f = 70, 16, 4, 384, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=90 + wd, bias=True, residual=True,
                            expert_norm=True, wdtype=wd)
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, residual=_cuda(lay)["residual"])
    print("expert norm", wd, "rel-L2", err)


def test_awq_fold_invariance_on_gpu():
    """Per-channel power-of-two scales folded into (1+gamma2) and their
    inverse into the gate_up columns give bit-identical routing and output."""
    T, E, k, d, f = 64, 16, 2, 256, 64
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=23, expert_norm=True)
    lay["expert_gamma"] = torch.round(lay["expert_gamma"] * 256) / 256
    s = torch.pow(2.0, torch.randint(-3, 4, (d,), generator=torch.Generator().manual_seed(6))
                  .double())
    lay2 = dict(lay)
    lay2["expert_gamma"] = ((1.0 + lay["expert_gamma"].double()) * s - 1.0).float()
    lay2["w_gate_up"] = (lay["w_gate_up"].double() / s).to(torch.bfloat16)
    outs = []
    for ly in (lay, lay2):
        g = _cuda(ly)
        layer = moe.MoeLayer(E, k, d, f)
        try:
            outs.append(run_gpu(layer, g, T).clone())
        finally:
            layer.close()
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("chunk", [0, 128])
def test_hot_expert_multi_chunk(chunk):
    """One expert receives every token (T=600 > 256): its work splits into
    three chunks of at most 256 tokens (the default above 256 tokens; the
    widest B stage is exercised), or five of at most 128."""
    T, E, k, d, f = 600, 16, 2, 256, 128
    lay = inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=77, bias=True)
    lay["router_bias"] = torch.zeros(E)
    lay["router_bias"][5] = 50.0
    err, _ = full_check(lay, _cuda(lay), E, k, d, f, options={moe.MOE_OPT_CHUNK_TOKENS: chunk})
    print("hot expert rel-L2", chunk, err)


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


def test_chunk_option_values():
    """MOE_OPT_CHUNK_TOKENS takes 0, 128 or 256 and nothing else."""
    layer = moe.MoeLayer(16, 2, 256, 64)
    try:
        for v in (0, 128, 256):
            assert moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_CHUNK_TOKENS, v,
                                           check=False) == moe.MOE_OK
        for v in (64, 100, 512, -1):
            assert moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_CHUNK_TOKENS, v,
                                           check=False) == moe.MOE_ERR_INVALID_ARG
    finally:
        layer.close()


def test_invalid_arguments_launch_nothing():
    T, E, k, d, f = 8, 16, 2, 256, 64
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=1))
    layer = moe.MoeLayer(E, k, d, f)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    args = [lay["x"], lay["router_w"], lay["router_gamma"], None, lay["w_gate_up"],
            lay["w_down"], None, None, None, out]  # expert_gamma passed by keyword (None)

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


def test_stack30_denoising_step_teacher_forced():
    """The 30-layer denoising step (distinct weights, Zipf(1.1)-skewed router
    bias, residual chained: x_{l+1} = x_l + MoE_l(x_l)).  Every layer is
    checked teacher-forced: the oracle gets the GPU's bf16 input of that
    layer, on 16 sampled tokens.  The chained output must match, and so must
    the layer's delta, run again on the GPU with the residual off and held to
    the parity tolerance on its own."""
    w = inputs.WORKLOADS["stack30"]
    x0 = inputs.make_layer(w, device="cuda")["x"]
    layer = moe.MoeLayer(w.E, w.k, w.d, w.f)
    xs = [x0]
    loads = []
    rows = np.random.default_rng(30).choice(w.T, 16, replace=False)
    deltas = []  # each layer's MoE output alone (residual off), sampled rows
    try:
        for l in range(w.layers):
            lay = inputs.make_layer(w, layer=l, device="cuda", with_x=False)
            nxt = torch.empty_like(x0)
            layer.forward(xs[-1], lay["router_w"], lay["router_gamma"], lay["w_gate_up"],
                          lay["w_down"], router_bias=lay["router_bias"], residual=xs[-1],
                          out=nxt, expert_gamma=lay["expert_gamma"])
            off, _, _ = layer.routing_tables(w.T)
            loads.append((off[1:] - off[:-1]).cpu())
            dl = torch.empty_like(x0)
            layer.forward(xs[-1], lay["router_w"], lay["router_gamma"], lay["w_gate_up"],
                          lay["w_down"], router_bias=lay["router_bias"], out=dl,
                          expert_gamma=lay["expert_gamma"])
            deltas.append(dl.cpu()[rows])
            xs.append(nxt)
            del lay
        assert layer.sync_status() == moe.MOE_OK
    finally:
        layer.close()
    worst, worst_d = 0.0, 0.0
    for l in range(w.layers):
        lay = _cpu(inputs.make_layer(w, layer=l, device="cuda", with_x=False))
        xin = xs[l].cpu()[rows]
        delta_ref, oidx, ow, ogap = oracle.moe_forward(
            xin, lay["router_w"], lay["router_gamma"], lay["router_bias"], lay["w_gate_up"],
            lay["w_down"], w.k, expert_gamma=lay["expert_gamma"])
        ref = xin.double().numpy() + delta_ref
        got = xs[l + 1].cpu()[rows].double().numpy()
        # out = bf16(x + delta) against the oracle's x + delta
        err = rel_l2(got, ref)
        assert err <= TOL_BF16, f"layer {l}: rel-L2 {err}"
        # the layer's delta, computed on the GPU with the residual off (so no
        # rounding of x + delta hides an error in it), at the parity tolerance
        derr = rel_l2(deltas[l].double().numpy(), delta_ref)
        assert derr <= TOL_BF16, f"layer {l}: delta rel-L2 {derr}"
        worst, worst_d = max(worst, err), max(worst_d, derr)
        del lay
    # the Zipf-skewed bias concentrates load: the busiest expert of each layer
    # takes several times the mean share
    ratio = max(float(c.max()) / float(c.float().mean()) for c in loads)
    assert ratio > 2.0
    print("stack30 worst layer rel-L2", worst, "worst delta rel-L2", worst_d,
          "max load / mean", ratio)


def test_cuda_graph_capture_replays_bit_identical():
    """Two chained layers (the second reads the first's output as x and as
    its residual) captured in one CUDA graph and replayed: the same bytes as
    the direct calls.  The calls allocate nothing once the workspace is
    reserved and never synchronise the host, so they capture as they are."""
    T, E, k, d, f = 96, 16, 4, 256, 128
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=515, bias=True))
    layer = moe.MoeLayer(E, k, d, f)
    try:
        moe.moe_plan_reserve(layer.plan, T)
        x = lay["x"]
        mid = torch.empty_like(x)
        out = torch.empty_like(x)

        def two_layers():
            layer.forward(x, lay["router_w"], lay["router_gamma"], lay["w_gate_up"],
                          lay["w_down"], router_bias=lay["router_bias"], out=mid)
            layer.forward(mid, lay["router_w"], lay["router_gamma"], lay["w_gate_up"],
                          lay["w_down"], router_bias=lay["router_bias"], residual=mid, out=out)

        two_layers()  # warm-up: one-time host queries happen outside the capture
        torch.cuda.synchronize()
        want_mid, want = mid.clone(), out.clone()
        mid.zero_()
        out.zero_()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                two_layers()
        torch.cuda.current_stream().wait_stream(s)
        for _ in range(3):
            mid.zero_()
            out.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(mid, want_mid)
            assert torch.equal(out, want)
        assert layer.sync_status() == moe.MOE_OK
        del g
    finally:
        layer.close()


def test_token_limits_launch_nothing():
    """T above MOE_MAX_T, or T * k above MOE_MAX_ASSIGNMENTS, is refused from
    the count alone: MOE_ERR_UNSUPPORTED, no workspace growth, no launch."""
    T, E, k, d, f = 8, 16, 16, 256, 64
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=4))
    layer = moe.MoeLayer(E, k, d, f)
    out = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    args = [lay["x"], lay["router_w"], lay["router_gamma"], None, lay["w_gate_up"],
            lay["w_down"], None, None, None, out]
    try:
        big_k = moe.MOE_MAX_ASSIGNMENTS // k + 1  # T * k over the limit, T itself allowed
        assert big_k <= moe.MOE_MAX_T
        for bad_T in (moe.MOE_MAX_T + 1, big_k, 2 ** 31 - 1):
            assert moe.moe_forward(layer.plan, bad_T, *args, check=False) == \
                moe.MOE_ERR_UNSUPPORTED
            assert moe.moe_plan_reserve(layer.plan, bad_T, check=False) == \
                moe.MOE_ERR_UNSUPPORTED
            st = moe.moe_route(layer.plan, bad_T, lay["x"], lay["router_w"], lay["router_gamma"],
                               None, out, out, None, check=False)
            assert st == moe.MOE_ERR_UNSUPPORTED
        torch.cuda.synchronize()
        assert torch.count_nonzero(out) == 0
        assert moe.moe_forward(layer.plan, T, *args, check=False) == moe.MOE_OK
        assert layer.sync_status() == moe.MOE_OK
    finally:
        layer.close()


def test_workspace_growth_is_refused_inside_a_capture():
    """A call that would grow the workspace while its stream is capturing
    returns MOE_ERR_UNSUPPORTED (no allocation node enters the graph); after
    moe_plan_reserve the same call captures."""
    T, E, k, d, f = 40, 16, 2, 256, 64
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=5))
    layer = moe.MoeLayer(E, k, d, f)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    args = [lay["x"], lay["router_w"], lay["router_gamma"], None, lay["w_gate_up"],
            lay["w_down"], None, None, None, out]
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                st = moe.moe_forward(layer.plan, T, *args, stream=s, check=False)
        assert st == moe.MOE_ERR_UNSUPPORTED
        del g
        moe.moe_plan_reserve(layer.plan, T)
        want = torch.empty_like(out)
        moe.moe_forward(layer.plan, T, *args[:-1], want)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                st = moe.moe_forward(layer.plan, T, *args, stream=s, check=False)
        assert st == moe.MOE_OK
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, want)
        assert layer.sync_status() == moe.MOE_OK
        del g
    finally:
        layer.close()


@pytest.mark.parametrize("wd", [inputs.WDTYPE_BF16, inputs.WDTYPE_INT4, inputs.WDTYPE_FP8,
                                inputs.WDTYPE_FP4])
def test_debug_guards_stay_intact(wd):
    """MOE_OPT_DEBUG: a guard block after every workspace region; ragged shapes
    through every weight format leave all guards intact (no kernel writes past
    its region) and give the same bytes as a plan without guards."""
    T, E, k, d, f = 77, 24, 5, 384, 192
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=31 + wd, wdtype=wd, bias=True,
                                  residual=True, expert_norm=True))
    outs = []
    for dbg in (0, 1):
        layer = moe.MoeLayer(E, k, d, f, wd)
        try:
            moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_DEBUG, dbg)
            for _ in range(2):
                o = run_gpu(layer, lay, T, residual=lay["residual"])
            outs.append(o.clone())
        finally:
            layer.close()
    assert torch.equal(outs[0], outs[1])
