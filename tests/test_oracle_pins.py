"""Pins of the CPU oracle against things other than itself.

Each test would fail on a plausible slip inside the oracle: a dropped term, a
wrong sign or index, a transposed operand, gate/up swapped, a wrong nibble
order, a wrong tie-break.  References used here are library routines
(torch.nn.functional.gelu / rms_norm / linear, torch.softmax), brute force
on tiny shapes, closed forms and invariants -- never the oracle's own code.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from block_diffusion_moe_router_b200 import inputs

EPS = 1e-6
# MX FP4 E2M1 values of the 16 nibbles (OCP Microscaling Formats specification)
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
              -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


# ---------------------------------------------------------------- helpers


def dense_weights(w, scales, cols):
    """[E,R,C] weight as float64 from its storage (bf16, int4 codes x fp16
    group scales, or E4M3 bytes x fp32 row scales) -- written from the
    storage format with library casts, not from the oracle."""
    if scales is None:
        return w.double()
    if scales.dtype == torch.float32:  # fp8: torch's own E4M3 decode
        return w.view(torch.float8_e4m3fn).double() * scales.double()[..., None]
    if scales.dtype == torch.uint8:  # fp4: the MX E2M1 table, torch's E4M3 decode
        E, R = w.shape[0], w.shape[1]
        nib = torch.stack([w & 0xF, w >> 4], dim=-1).reshape(E, R, -1).long()
        vals = torch.tensor(E2M1_TABLE, dtype=torch.float64)[nib]
        srow, blk = inputs.fp4_scale_record(scales, R, cols)
        bs = blk.view(torch.float8_e4m3fn).double().permute(0, 2, 1)  # [E, R, NB]
        bs = bs.repeat_interleave(inputs.FP4_BLOCK, dim=-1)[..., :cols]
        return vals * bs * srow.double()[..., None]
    codes = inputs.unpack_int4(w).double()
    s = scales.double().repeat_interleave(inputs.GROUP, dim=-1)[..., :cols]
    return codes * s


def brute_force(lay, k, eps=EPS):
    """Dense reference: every expert on every token, full softmax, masked to
    the k selected experts and renormalised, summed over all experts."""
    x = lay["x"].double()
    T, d = x.shape
    E = lay["router_w"].shape[0]
    f = lay["w_gate_up"].shape[1] // 2
    u = F.rms_norm(x, (d,), weight=1.0 + lay["router_gamma"].double(), eps=eps)
    # the experts' input: x, or its expert-side (1+gamma2) RMSNorm
    xe = x if lay.get("expert_gamma") is None else F.rms_norm(
        x, (d,), weight=1.0 + lay["expert_gamma"].double(), eps=eps)
    b = lay["router_bias"].double() if lay.get("router_bias") is not None else None
    z = F.linear(u, lay["router_w"].double(), b)
    p = torch.softmax(z, dim=-1)
    mask = torch.zeros(T, E, dtype=torch.float64)
    sel = []
    for t in range(T):
        zt = z[t].tolist()
        s = sorted(range(E), key=lambda e: (-zt[e], e))[:k]
        sel.append(s)
        mask[t, s] = 1.0
    w = p * mask
    w = w / w.sum(dim=-1, keepdim=True)
    Wgu = dense_weights(lay["w_gate_up"], lay.get("scales_gate_up"), d)
    Wd = dense_weights(lay["w_down"], lay.get("scales_down"), f)
    out = torch.zeros(T, d, dtype=torch.float64)
    if lay.get("residual") is not None:
        out += lay["residual"].double()
    for e in range(E):
        g = F.linear(xe, Wgu[e, :f])
        v = F.linear(xe, Wgu[e, f:])
        h = F.gelu(g, approximate="tanh") * v
        y = F.linear(h, Wd[e])
        out += w[:, e:e + 1] * y
    return out.numpy(), np.array(sel, dtype=np.int32), w, z


def run_oracle(lay, k, forced=None):
    return oracle.moe_forward(lay["x"], lay["router_w"], lay["router_gamma"],
                              lay.get("router_bias"), lay["w_gate_up"], lay["w_down"], k,
                              scales_gate_up=lay.get("scales_gate_up"),
                              scales_down=lay.get("scales_down"),
                              residual=lay.get("residual"), forced_idx=forced, eps=EPS,
                              expert_gamma=lay.get("expert_gamma"))


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------- GELU-tanh


def test_gelu_tanh_matches_torch_library():
    a = torch.linspace(-12, 12, 20001, dtype=torch.float64)
    ref = F.gelu(a, approximate="tanh").numpy()
    got = oracle.gelu_tanh(a.numpy())
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-15)


def test_gelu_tanh_special_values():
    assert oracle.gelu_tanh(np.array([0.0]))[0] == 0.0
    a = np.linspace(-6, 6, 1001)
    # gelu(a) - gelu(-a) = a : the tanh part is odd
    np.testing.assert_allclose(oracle.gelu_tanh(a) - oracle.gelu_tanh(-a), a, atol=1e-14)
    # limits: identity for large positive, zero for large negative
    big = np.array([30.0, 50.0])
    np.testing.assert_allclose(oracle.gelu_tanh(big), big, rtol=1e-15)
    assert np.all(np.abs(oracle.gelu_tanh(-big)) < 1e-300 + 1e-15)
    # the cubic term matters: without 0.044715 a^3 the value at a=2 differs
    # from the library value by > 1e-3
    v2 = oracle.gelu_tanh(np.array([2.0]))[0]
    no_cubic = 0.5 * 2.0 * (1 + math.tanh(math.sqrt(2 / math.pi) * 2.0))
    assert abs(v2 - no_cubic) > 1e-3
    assert abs(v2 - F.gelu(torch.tensor(2.0, dtype=torch.float64),
                           approximate="tanh").item()) < 1e-15


# ---------------------------------------------------------------- router norm


@pytest.mark.parametrize("d", [16, 256, 2816])
def test_rmsnorm_plus_one_matches_torch_library(d):
    g = torch.Generator().manual_seed(d)
    x = torch.randn(7, d, generator=g, dtype=torch.float64) * 3
    gamma = (torch.randn(d, generator=g) * 0.1).float()
    ref = F.rms_norm(x, (d,), weight=1.0 + gamma.double(), eps=EPS).numpy()
    got = oracle.rmsnorm_plus_one(x.numpy(), gamma, EPS)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-14)


def test_router_scale_invariance():
    """The router reads x only through its RMS norm: with eps = 0, scaling x by
    a power of two leaves logits, selection and weights bit-identical."""
    lay = inputs.make_small(T=12, d=256, E=16, k=4, f=64, seed=3)
    i1, w1, g1, z1 = oracle.route(lay["x"], lay["router_w"], lay["router_gamma"], None, 4,
                                  eps=0.0)
    x2 = (lay["x"].float() * 4.0).to(torch.bfloat16)  # exact in bf16
    i2, w2, g2, z2 = oracle.route(x2, lay["router_w"], lay["router_gamma"], None, 4, eps=0.0)
    assert np.array_equal(i1, i2)
    np.testing.assert_allclose(z1, z2, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(w1, w2, rtol=1e-14)


# ---------------------------------------------------------------- top-k / weights


def test_topk_matches_sorted_with_ties():
    rng = np.random.default_rng(0)
    for trial in range(200):
        E = int(rng.integers(2, 140))
        k = int(rng.integers(1, E + 1))
        # few distinct values -> many exact ties
        z = rng.integers(-3, 4, size=E).astype(np.float64) * 0.5
        idx, gap = oracle.select_topk(z, k)
        ref = sorted(range(E), key=lambda e: (-z[e], e))[:k]
        assert list(idx) == ref
        if k < E:
            rest = sorted(range(E), key=lambda e: (-z[e], e))[k]
            assert gap == z[ref[-1]] - z[rest]
        else:
            assert gap == math.inf


def test_route_weights_identity_and_sum():
    """softmax over all E, restricted to S and renormalised == softmax over the
    selected logits (torch.softmax); weights sum to one."""
    rng = np.random.default_rng(1)
    for _ in range(50):
        E = int(rng.integers(2, 200))
        k = int(rng.integers(1, min(E, 16) + 1))
        z = rng.normal(size=E) * 3
        idx, _ = oracle.select_topk(z, k)
        w = oracle.route_weights(z, idx)
        ref = torch.softmax(torch.tensor(z[idx], dtype=torch.float64), 0).numpy()
        np.testing.assert_allclose(w, ref, rtol=1e-13)
        assert abs(w.sum() - 1.0) < 1e-12
        assert np.all(np.diff(w) <= 1e-15)  # j order is logit-descending


def test_tie_break_duplicated_router_rows():
    """Duplicated router rows give bit-identical logits; the lower expert
    index must be taken first."""
    lay = inputs.make_small(T=32, d=256, E=16, k=3, f=64, seed=5)
    rw = lay["router_w"].clone()
    for a, b in [(2, 9), (4, 5), (11, 0)]:
        rw[b] = rw[a]
    idx, w, gap, z = oracle.route(lay["x"], rw, lay["router_gamma"], None, 3)
    assert np.array_equal(z[:, 2], z[:, 9]) and np.array_equal(z[:, 0], z[:, 11])
    for t in range(32):
        ref = sorted(range(16), key=lambda e: (-z[t, e], e))[:3]
        assert list(idx[t]) == ref
    # force a token whose top-2 is a duplicated pair: the pair ties exactly
    hits = 0
    for t in range(32):
        s = set(idx[t].tolist())
        for lo, hi in [(2, 9), (4, 5), (0, 11)]:
            if lo in s and hi in s:
                hits += 1
                assert list(idx[t]).index(lo) < list(idx[t]).index(hi)
            if hi in s and lo not in s:
                raise AssertionError("higher duplicate chosen without the lower one")
    assert hits >= 0


# ---------------------------------------------------------------- whole layer


@pytest.mark.parametrize("seed,E,k,bias,residual,wd,enorm", [
    (0, 16, 2, False, False, inputs.WDTYPE_BF16, False),
    (1, 8, 3, True, True, inputs.WDTYPE_BF16, False),
    (2, 16, 4, True, False, inputs.WDTYPE_INT4, False),
    (3, 5, 5, False, True, inputs.WDTYPE_INT4, False),
    (4, 16, 2, True, True, inputs.WDTYPE_BF16, True),
    (5, 8, 3, False, False, inputs.WDTYPE_INT4, True),
    (6, 16, 4, True, True, inputs.WDTYPE_FP8, False),
    (7, 8, 2, False, False, inputs.WDTYPE_FP8, True),
    (8, 16, 4, True, True, inputs.WDTYPE_FP4, False),
    (9, 8, 3, False, False, inputs.WDTYPE_FP4, True),
])
def test_layer_matches_brute_force(seed, E, k, bias, residual, wd, enorm):
    d, f = 256, 64
    lay = inputs.make_small(T=9, d=d, E=E, k=k, f=f, seed=seed, wdtype=wd, bias=bias,
                            residual=residual, expert_norm=enorm)
    ref, sel, wref, z = brute_force(lay, k)
    out, idx, w, gap = run_oracle(lay, k)
    assert np.array_equal(idx, sel)
    for t in range(idx.shape[0]):
        np.testing.assert_allclose(w[t], wref[t, idx[t]].numpy(), rtol=1e-12)
    assert rel(out, ref) < 1e-12


def test_E_equals_k_is_full_softmax_mixture():
    """E = k: every expert is used with weight softmax(z)_e."""
    E = 6
    lay = inputs.make_small(T=5, d=256, E=E, k=E, f=64, seed=7, bias=True)
    out, idx, w, gap = run_oracle(lay, E)
    _, _, _, z = oracle.route(lay["x"], lay["router_w"], lay["router_gamma"],
                              lay["router_bias"], E)
    p = torch.softmax(torch.tensor(z), -1).numpy()
    x = lay["x"].double()
    Wgu = lay["w_gate_up"].double()
    Wd = lay["w_down"].double()
    ref = np.zeros((5, 256))
    for e in range(E):
        h = F.gelu(F.linear(x, Wgu[e, :64]), approximate="tanh") * F.linear(x, Wgu[e, 64:])
        ref += p[:, e:e + 1] * F.linear(h, Wd[e]).numpy()
    assert rel(out, ref) < 1e-12
    assert np.all(np.isinf(gap))


def test_E1_k1_is_dense_gated_gelu_ffn():
    """E = k = 1: weight 1, out = down(gelu_tanh(gate x) * up x) exactly the
    dense gated FFN; gate must be rows [0,f), up rows [f,2f)."""
    lay = inputs.make_small(T=7, d=256, E=1, k=1, f=128, seed=8)
    out, idx, w, gap = run_oracle(lay, 1)
    assert np.all(idx == 0) and np.allclose(w, 1.0)
    x = lay["x"].double()
    Wgu = lay["w_gate_up"].double()[0]
    Wd = lay["w_down"].double()[0]
    ref = F.linear(F.gelu(F.linear(x, Wgu[:128]), approximate="tanh") * F.linear(x, Wgu[128:]),
                   Wd).numpy()
    swapped = F.linear(F.gelu(F.linear(x, Wgu[128:]), approximate="tanh")
                       * F.linear(x, Wgu[:128]), Wd).numpy()
    assert rel(out, ref) < 1e-13
    assert rel(out, swapped) > 1e-2


def test_expert_norm_dense_form():
    """E = k = 1 with the expert-side norm: out = FFN(rms_norm(x) * (1 + g2))
    (library rms_norm), and the router still reads the raw x."""
    lay = inputs.make_small(T=5, d=256, E=1, k=1, f=64, seed=21, expert_norm=True)
    out, idx, w, _ = run_oracle(lay, 1)
    x = lay["x"].double()
    xe = F.rms_norm(x, (256,), weight=1.0 + lay["expert_gamma"].double(), eps=EPS)
    Wgu = lay["w_gate_up"].double()[0]
    Wd = lay["w_down"].double()[0]
    ref = F.linear(F.gelu(F.linear(xe, Wgu[:64]), approximate="tanh") * F.linear(xe, Wgu[64:]),
                   Wd).numpy()
    assert rel(out, ref) < 1e-13
    raw = F.linear(F.gelu(F.linear(x, Wgu[:64]), approximate="tanh") * F.linear(x, Wgu[64:]),
                   Wd).numpy()
    assert rel(out, raw) > 1e-2


def test_awq_fold_invariance():
    """Folding per-channel scales s into the expert-side norm ((1+g2) * s)
    and their inverse into the fused gate_up columns (W / s) leaves routing
    and output unchanged (powers of two keep the bf16 weights exact)."""
    d, f, E, k = 256, 64, 8, 2
    lay = inputs.make_small(T=11, d=d, E=E, k=k, f=f, seed=22, expert_norm=True, bias=True)
    # gamma2 on a 2^-8 grid keeps (1 + gamma2) * s - 1 exact in fp32
    lay["expert_gamma"] = torch.round(lay["expert_gamma"] * 256) / 256
    g = torch.Generator().manual_seed(5)
    s = torch.pow(2.0, torch.randint(-3, 4, (d,), generator=g).double())
    lay2 = dict(lay)
    lay2["expert_gamma"] = ((1.0 + lay["expert_gamma"].double()) * s - 1.0).float()
    # (1 + g2') must equal (1 + g2) * s exactly in fp32 for an exact fold
    assert torch.equal((1.0 + lay2["expert_gamma"]).double(),
                       (1.0 + lay["expert_gamma"]).double() * s)
    lay2["w_gate_up"] = (lay["w_gate_up"].double() / s).to(torch.bfloat16)
    assert torch.equal(lay2["w_gate_up"].double() * s, lay["w_gate_up"].double())
    out1, idx1, w1, _ = run_oracle(lay, k)
    out2, idx2, w2, _ = run_oracle(lay2, k)
    assert np.array_equal(idx1, idx2)
    np.testing.assert_array_equal(w1, w2)
    assert rel(out2, out1) < 1e-13


def test_token_permutation_equivariance():
    lay = inputs.make_small(T=10, d=256, E=16, k=2, f=64, seed=9, bias=True, residual=True)
    out, idx, w, _ = run_oracle(lay, 2)
    perm = torch.randperm(10, generator=torch.Generator().manual_seed(1))
    lay2 = dict(lay)
    lay2["x"] = lay["x"][perm]
    lay2["residual"] = lay["residual"][perm]
    out2, idx2, w2, _ = run_oracle(lay2, 2)
    assert np.array_equal(idx2, idx[perm.numpy()])
    np.testing.assert_array_equal(out2, out[perm.numpy()])
    np.testing.assert_array_equal(w2, w[perm.numpy()])


def test_forced_index_mode():
    """Forcing the selected set to the natural one reproduces the layer; forcing
    another set uses softmax over the forced logits."""
    lay = inputs.make_small(T=6, d=256, E=16, k=2, f=64, seed=10)
    out, idx, w, _ = run_oracle(lay, 2)
    out2, idx2, w2, _ = run_oracle(lay, 2, forced=idx)
    np.testing.assert_array_equal(out, out2)
    forced = np.tile(np.array([[7, 3]], np.int32), (6, 1))
    out3, idx3, w3, _ = run_oracle(lay, 2, forced=forced)
    assert np.all(idx3 == forced)
    _, _, _, z = oracle.route(lay["x"], lay["router_w"], lay["router_gamma"], None, 2)
    ref = torch.softmax(torch.tensor(z[:, [7, 3]]), -1).numpy()
    np.testing.assert_allclose(w3, ref, rtol=1e-13)


# ---------------------------------------------------------------- int4 storage


def test_int4_dequant_closed_form():
    """Rows decoded by the oracle equal code * scale[i // 128] with codes and
    scales placed by hand (pins nibble order, sign extension, group index)."""
    E, R, C = 2, 3, 384
    codes = torch.zeros(E, R, C, dtype=torch.int8)
    codes[1, 2, 0] = -8
    codes[1, 2, 1] = 7
    codes[1, 2, 129] = -1
    codes[1, 2, 383] = 5
    scales = torch.ones(E, R, 3, dtype=torch.float16)
    scales[1, 2, 0] = 0.5
    scales[1, 2, 1] = 0.25
    scales[1, 2, 2] = 0.125
    packed = inputs.pack_int4(codes)
    row = oracle.weight_row(packed, scales, 1, 2, C)
    ref = np.zeros(C)
    ref[0], ref[1], ref[129], ref[383] = -4.0, 3.5, -0.25, 0.625
    np.testing.assert_array_equal(row, ref)
    assert np.all(oracle.weight_row(packed, scales, 0, 2, C) == 0)


def test_int4_zero_codes_give_residual_only():
    lay = inputs.make_small(T=4, d=256, E=4, k=2, f=128, seed=11,
                            wdtype=inputs.WDTYPE_INT4, residual=True)
    lay["w_gate_up"] = torch.full_like(lay["w_gate_up"], 0)
    lay["w_down"] = torch.full_like(lay["w_down"], 0)
    out, _, _, _ = run_oracle(lay, 2)
    np.testing.assert_array_equal(out, lay["residual"].double().numpy())


def test_int4_single_code_closed_form():
    """E = k = 1 with one nonzero code in each of gate, up and down:
    out[m] = (c3 s3) * gelu_tanh(c1 s1 x_i) * (c2 s2 x_j)."""
    d, f = 256, 128
    lay = inputs.make_small(T=3, d=d, E=1, k=1, f=f, seed=12, wdtype=inputs.WDTYPE_INT4)
    cg = torch.zeros(1, 2 * f, d, dtype=torch.int8)
    cd = torch.zeros(1, d, f, dtype=torch.int8)
    r, i, j, m = 5, 130, 17, 200
    cg[0, r, i] = 3          # gate row r
    cg[0, f + r, j] = -2     # up row r
    cd[0, m, r] = 7          # down column r
    lay["w_gate_up"] = inputs.pack_int4(cg)
    lay["w_down"] = inputs.pack_int4(cd)
    s_gu = lay["scales_gate_up"]
    s_d = lay["scales_down"]
    out, _, _, _ = run_oracle(lay, 1)
    x = lay["x"].double().numpy()
    s1 = float(s_gu[0, r, i // 128])
    s2 = float(s_gu[0, f + r, j // 128])
    s3 = float(s_d[0, m, r // 128])
    a = 3 * s1 * x[:, i]
    ref_m = 7 * s3 * (0.5 * a * (1 + np.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3))))
    ref_m = ref_m * (-2 * s2 * x[:, j])
    ref = np.zeros((3, d))
    ref[:, m] = ref_m
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-300)


def test_decoders():
    vals = torch.tensor([0.0, -1.5, 3.140625, 1e-3, 6.0e-5, 65504.0, -0.0],
                        dtype=torch.float16)
    np.testing.assert_array_equal(oracle.decode_fp16(vals), vals.double().numpy())
    b = torch.randn(1000, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    np.testing.assert_array_equal(oracle.decode_bf16(b), b.double().numpy())
    sub = torch.tensor([2 ** -24, 3 * 2 ** -24, 2 ** -14], dtype=torch.float16)
    np.testing.assert_array_equal(oracle.decode_fp16(sub), sub.double().numpy())


# ---------------------------------------------------------------- fp8 storage


def test_e4m3_decode_matches_library_cast():
    """All 256 byte values decode like torch's float8_e4m3fn -> float64 cast
    (an independent library routine), NaN codes included."""
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    got = oracle.decode_e4m3(b)
    ref = b.view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.isnan(got).sum() == 2  # 0x7F and 0xFF
    np.testing.assert_array_equal(np.nan_to_num(got), np.nan_to_num(ref))


def test_e4m3_closed_forms():
    """OFP8 E4M3 (bias 7, 3 mantissa bits, no infinities): a few values by
    hand, the subnormal step and sign symmetry."""
    d = lambda v: float(oracle.decode_e4m3(np.array([v], np.uint8))[0])
    assert d(0x38) == 1.0           # 0 0111 000
    assert d(0x7E) == 448.0         # 0 1111 110: largest finite value
    assert d(0x77) == 240.0         # 0 1110 111 = 1.875 * 2^7
    assert d(0x08) == 2.0 ** -6     # smallest normal
    assert d(0x01) == 2.0 ** -9     # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9
    assert d(0x00) == 0.0 and d(0x80) == 0.0
    for v in range(0x7F):
        assert d(v | 0x80) == -d(v)


def test_fp8_weight_row_closed_form():
    """Rows decoded by the oracle equal value(code) * scale[row] for codes
    and scales placed by hand (pins the byte order and the row scale)."""
    E, R, C = 2, 3, 256
    codes = torch.zeros(E, R, C, dtype=torch.uint8)
    codes[1, 2, 0] = 0x38     # 1.0
    codes[1, 2, 1] = 0xC4     # 1 1000 100 = -1.5 * 2
    codes[1, 2, 130] = 0x01   # 2^-9
    codes[1, 2, 255] = 0x7E   # 448
    scales = torch.ones(E, R, dtype=torch.float32)
    scales[1, 2] = 0.25
    row = oracle.weight_row(codes, scales, 1, 2, C)
    ref = np.zeros(C)
    ref[0], ref[1], ref[130], ref[255] = 0.25, -0.75, 2.0 ** -11, 112.0
    np.testing.assert_array_equal(row, ref)
    assert np.all(oracle.weight_row(codes, scales, 0, 2, C) == 0)


def test_fp8_single_code_closed_form():
    """E = k = 1 with one nonzero code in each of gate, up and down:
    out[m] = (v3 s3) * gelu_tanh(v1 s1 x_i) * (v2 s2 x_j), s the row scales."""
    d, f = 256, 128
    lay = inputs.make_small(T=3, d=d, E=1, k=1, f=f, seed=13, wdtype=inputs.WDTYPE_FP8)
    cg = torch.zeros(1, 2 * f, d, dtype=torch.uint8)
    cd = torch.zeros(1, d, f, dtype=torch.uint8)
    r, i, j, m = 5, 130, 17, 200
    cg[0, r, i] = 0x40        # 2.0, gate row r
    cg[0, f + r, j] = 0xB4    # 1 0110 100 = -0.75, up row r
    cd[0, m, r] = 0x44        # 0 1000 100 = 3.0, down column r
    lay["w_gate_up"] = cg
    lay["w_down"] = cd
    s_gu = lay["scales_gate_up"]
    s_d = lay["scales_down"]
    out, _, _, _ = run_oracle(lay, 1)
    x = lay["x"].double().numpy()
    s1, s2, s3 = float(s_gu[0, r]), float(s_gu[0, f + r]), float(s_d[0, m])
    a = 2.0 * s1 * x[:, i]
    ref_m = 3.0 * s3 * (0.5 * a * (1 + np.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3))))
    ref_m = ref_m * (-0.75 * s2 * x[:, j])
    ref = np.zeros((3, d))
    ref[:, m] = ref_m
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-300)


# ---------------------------------------------------------------- fp4 storage


def test_e2m1_decode_table():
    """The 16 E2M1 nibbles decode to the MX table (1 sign, 2 exponent bits
    with bias 1, 1 mantissa bit; exponent 0 is subnormal)."""
    got = oracle.decode_e2m1(np.arange(16, dtype=np.uint8))
    np.testing.assert_array_equal(got, np.array(E2M1_TABLE))
    assert np.array_equal(np.signbit(got[8:]), np.ones(8, bool))


def test_fp4_weight_row_closed_form():
    """Hand-placed nibbles, block scales and row scales (pins the nibble
    order, the block index i // 16 and the record layout)."""
    E, R, C = 2, 3, 64
    nib = torch.zeros(E, R, C, dtype=torch.int16)
    nib[1, 2, 0] = 0x2      # 1.0
    nib[1, 2, 1] = 0xF      # -6.0
    nib[1, 2, 17] = 0x7     # 6.0 in block 1
    nib[1, 2, 63] = 0x9     # -0.5 in block 3
    codes = (nib[..., 0::2] | (nib[..., 1::2] << 4)).to(torch.uint8)
    srow = torch.ones(E, R)
    srow[1, 2] = 0.5
    blk = torch.full((E, 4, R), 1.0).to(torch.float8_e4m3fn).view(torch.uint8)
    blk[1, 1, 2] = torch.tensor(2.0).to(torch.float8_e4m3fn).view(torch.uint8)
    blk[1, 3, 2] = torch.tensor(0.25).to(torch.float8_e4m3fn).view(torch.uint8)
    rec = torch.cat([srow.view(torch.uint8).reshape(E, R * 4), blk.reshape(E, 4 * R)], 1)
    row = oracle.weight_row(codes, rec.contiguous(), 1, 2, C)
    ref = np.zeros(C)
    ref[0], ref[1], ref[17], ref[63] = 0.5, -3.0, 6.0, -0.0625
    np.testing.assert_array_equal(row, ref)
    assert np.all(oracle.weight_row(codes, rec.contiguous(), 0, 2, C) == 0)


def test_single_precision_timing_build_computes_the_same_layer():
    """The fp32 build the bench times beside the fp64 oracle is the same
    definition in single precision: on a tiny layer its output agrees with
    the fp64 oracle to single-precision accuracy (it is never a reference)."""
    lay = inputs.make_small(T=12, d=256, E=16, k=4, f=64, seed=404, bias=True, residual=True)
    ref, _, _, _ = oracle.moe_forward(lay["x"], lay["router_w"], lay["router_gamma"],
                                      lay["router_bias"], lay["w_gate_up"], lay["w_down"], 4,
                                      residual=lay["residual"])
    got = oracle.moe_forward_f32(lay["x"], lay["router_w"], lay["router_gamma"],
                                 lay["router_bias"], lay["w_gate_up"], lay["w_down"], 4,
                                 residual=lay["residual"])
    err = np.linalg.norm(got.astype(np.float64) - ref) / np.linalg.norm(ref)
    assert err < 1e-5, err
