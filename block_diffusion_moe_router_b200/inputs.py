"""Seeded synthetic inputs for the top-k mixture-of-experts FFN layer.

This module only draws random tensors and packs integer codes into bytes.  It
holds none of the layer's arithmetic, so both the CUDA path and the CPU oracle
can consume its output without sharing any computation.

Workloads (shapes and distributions follow the DiffusionGemma 26B-A4B pages:
128 experts with 8 active per token, a 256-token canvas, hidden 2816 and
per-expert intermediate 704, symmetric int4 weights in groups of 128):

  tiny     T=16,   d=256,  E=16,  k=2, f=64,  bf16 weights
  canvas   T=256,  d=2816, E=128, k=8, f=704, bf16 weights
  canvas4  T=256,  d=2816, E=128, k=8, f=704, int4 w4g128 weights + fp16 scales
  canvas8  T=256,  d=2816, E=128, k=8, f=704, fp8 E4M3 weights + fp32 row scales
  canvas4f T=256,  d=2816, E=128, k=8, f=704, fp4 E2M1 weights + E4M3 block
           scales (16 elements) + fp32 row scales
  encode   T=2048, d=2816, E=128, k=8, f=704, bf16 weights (prompt + canvas)
  stack30  30 layers of `canvas`, distinct weights, Zipf(1.1)-skewed router bias,
           residual carried between layers, experts reading the (1+gamma2)
           RMSNorm of x (the model's pre-FFN norm; gamma2 ~ N(0, 0.1^2))

Distributions: x ~ N(0,1) rounded to bf16; router W ~ N(0, 1/d) (variance 1/d,
so logits have unit scale) in fp32; gamma ~ N(0, 0.1^2) in fp32; expert weights
~ N(0, 0.02^2) rounded to bf16; int4 codes uniform on [-8, 7] and scales
U(0.001, 0.01) rounded to fp16; fp8 codes: N(0, 64^2) draws clamped to
+-448 and rounded to E4M3 by torch's float8_e4m3fn cast (the codes span the
format, a few subnormals included), row scales U(0.5, 1.5) * 0.02 / 64 in
fp32 (so the weights are about N(0, 0.02^2) like the bf16 ones).
Seeds: 1000*workload_id + 10*layer + tensor_id.

Layouts (all row-major, contiguous):
  x            [T, d]            bf16
  router_w     [E, d]            fp32
  router_gamma [d]               fp32 (applied as 1 + gamma)
  router_bias  [E]               fp32 or None
  expert_gamma [d]               fp32 or None (experts read rmsnorm(x)*(1+gamma2))
  w_gate_up    [E, 2f, d]        bf16 (rows [0,f) gate, [f,2f) up)
               [E, 2f, d/2]      uint8 for int4 (element i in byte i/2, low
                                 nibble for even i, 4-bit two's complement)
               [E, 2f, d]        uint8 for fp8 (E4M3 bytes)
  w_down       [E, d, f]         bf16, or [E, d, f/2] uint8 for int4, or
                                 [E, d, f] uint8 for fp8
  scales_gu    [E, 2f, ceil(d/128)] fp16 (int4), [E, 2f] fp32 (fp8)
  scales_d     [E, d, ceil(f/128)]  fp16 (int4), [E, d] fp32 (fp8)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

GROUP = 128  # int4 quantisation group along the input dimension

WDTYPE_BF16 = 0
WDTYPE_INT4 = 1
WDTYPE_FP8 = 2
WDTYPE_FP4 = 3
FP4_BLOCK = 16        # elements per E4M3 block scale of the fp4 weights
FP8_CODE_STD = 64.0   # spread of the E4M3 code draws


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int          # workload id used in the seed formula
    T: int
    d: int
    E: int
    k: int
    f: int
    wdtype: int = WDTYPE_BF16
    layers: int = 1
    zipf_s: float = 0.0   # > 0: router bias drawn so expert load is Zipf(s)-skewed
    residual: bool = False
    expert_norm: bool = False  # experts read the (1+gamma2) RMSNorm of x
    act_wid: Optional[int] = None  # take x / router tensors from another workload's seeds

    @property
    def n_groups_d(self) -> int:
        return (self.d + GROUP - 1) // GROUP

    @property
    def n_groups_f(self) -> int:
        return (self.f + GROUP - 1) // GROUP


WORKLOADS = {
    "tiny": Workload("tiny", 0, T=16, d=256, E=16, k=2, f=64),
    "canvas": Workload("canvas", 1, T=256, d=2816, E=128, k=8, f=704),
    "canvas4": Workload("canvas4", 2, T=256, d=2816, E=128, k=8, f=704,
                        wdtype=WDTYPE_INT4, act_wid=1),
    "canvas8": Workload("canvas8", 5, T=256, d=2816, E=128, k=8, f=704,
                        wdtype=WDTYPE_FP8, act_wid=1),
    "canvas4f": Workload("canvas4f", 6, T=256, d=2816, E=128, k=8, f=704,
                         wdtype=WDTYPE_FP4, act_wid=1),
    "encode": Workload("encode", 3, T=2048, d=2816, E=128, k=8, f=704),
    "stack30": Workload("stack30", 4, T=256, d=2816, E=128, k=8, f=704,
                        layers=30, zipf_s=1.1, residual=True, expert_norm=True),
}

# tensor ids inside the seed formula
(_TID_X, _TID_RW, _TID_GAMMA, _TID_WGU, _TID_WD, _TID_SGU, _TID_SD, _TID_BIAS,
 _TID_EGAMMA) = range(9)


def seed_for(wid: int, layer: int, tensor_id: int) -> int:
    return 1000 * wid + 10 * layer + tensor_id


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, std, seed, device, dtype):
    g = _gen(seed, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def pack_int4(codes: torch.Tensor) -> torch.Tensor:
    """Pack int8 codes in [-8, 7] along the last dim: element i -> byte i/2,
    low nibble for even i (4-bit two's complement)."""
    assert codes.shape[-1] % 2 == 0
    c = codes.to(torch.int16) & 0xF
    lo = c[..., 0::2]
    hi = c[..., 1::2]
    return (lo | (hi << 4)).to(torch.uint8)


def unpack_int4(packed: torch.Tensor) -> torch.Tensor:
    """Inverse of pack_int4 (pure bit manipulation): uint8 -> int8 codes."""
    p = packed.to(torch.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    out = torch.stack([lo, hi], dim=-1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    out = torch.where(out >= 8, out - 16, out)
    return out.to(torch.int8)


def make_int4(shape, seed_codes, seed_scales, device):
    """Random int4 codes uniform on [-8, 7] (packed) and U(0.001, 0.01) fp16
    scales, one per group of 128 along the last (input) dimension."""
    E, rows, cols = shape
    g = _gen(seed_codes, device)
    codes = torch.randint(-8, 8, (E, rows, cols), generator=g, device=device, dtype=torch.int8)
    ng = (cols + GROUP - 1) // GROUP
    gs = _gen(seed_scales, device)
    scales = (torch.rand((E, rows, ng), generator=gs, device=device, dtype=torch.float32)
              * 0.009 + 0.001).to(torch.float16)
    return pack_int4(codes), scales


def make_fp8(shape, seed_codes, seed_scales, device):
    """Random E4M3 codes (uint8 bytes) and fp32 scales, one per row: the
    codes are N(0, 64^2) draws clamped to +-448 and rounded to E4M3 by
    torch's float8_e4m3fn cast (no NaN code can come out); the scales are
    U(0.5, 1.5) * 0.02 / 64."""
    E, rows, cols = shape
    v = _randn((E, rows, cols), FP8_CODE_STD, seed_codes, device, torch.float32)
    codes = v.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    gs = _gen(seed_scales, device)
    scales = (torch.rand((E, rows), generator=gs, device=device, dtype=torch.float32) + 0.5) \
        * (0.02 / FP8_CODE_STD)
    return codes, scales


def make_fp4(shape, seed_codes, seed_scales, device):
    """Random E2M1 codes (uniform over the 16 nibbles, packed two per byte
    like the int4 codes) and their scale records: per expert e, the fp32 row
    scales [R] (U(0.5, 1.5) * 0.01) then the E4M3 block scales [NB][R] (N(1,
    0.25^2) draws clamped to [0.25, 4] and rounded to E4M3 by torch's cast),
    NB = ceil(C/16), all as one uint8 tensor [E, 4R + NB R]."""
    E, rows, cols = shape
    g = _gen(seed_codes, device)
    nib = torch.randint(0, 16, (E, rows, cols), generator=g, device=device, dtype=torch.int16)
    codes = (nib[..., 0::2] | (nib[..., 1::2] << 4)).to(torch.uint8)
    nb = (cols + FP4_BLOCK - 1) // FP4_BLOCK
    gs = _gen(seed_scales, device)
    srow = (torch.rand((E, rows), generator=gs, device=device) + 0.5) * 0.01
    blk = (torch.randn((E, nb, rows), generator=gs, device=device) * 0.25 + 1.0).clamp_(0.25, 4.0)
    blk = blk.to(torch.float8_e4m3fn).view(torch.uint8)
    rec = torch.cat([srow.contiguous().view(torch.uint8).reshape(E, rows * 4),
                     blk.reshape(E, nb * rows)], dim=1)
    return codes, rec.contiguous()


def fp4_scale_record(rec: torch.Tensor, rows: int, cols: int):
    """Split scale records (see make_fp4) into fp32 row scales [E, R] and
    E4M3 block-scale bytes [E, NB, R] (byte reinterpretation only)."""
    E = rec.shape[0]
    nb = (cols + FP4_BLOCK - 1) // FP4_BLOCK
    srow = rec[:, :rows * 4].contiguous().view(torch.float32).reshape(E, rows)
    blk = rec[:, rows * 4:].reshape(E, nb, rows)
    return srow, blk


def zipf_bias(E: int, s: float, seed: int, device) -> torch.Tensor:
    """Router bias whose exp() follows a Zipf(s) law over a seeded random
    ranking of the experts: b_e = -s * ln(rank_e), rank_e in 1..E."""
    g = _gen(seed, "cpu")
    rank = torch.randperm(E, generator=g).to(torch.float64) + 1.0
    return (-s * torch.log(rank)).to(torch.float32).to(device)


def make_layer(w: Workload, layer: int = 0, device="cpu", T: Optional[int] = None,
               with_x: bool = True) -> dict:
    """All tensors of one layer of workload `w` (see module docstring)."""
    T = w.T if T is None else T
    awid = w.wid if w.act_wid is None else w.act_wid
    out = {}
    if with_x:
        out["x"] = _randn((T, w.d), 1.0, seed_for(awid, 0, _TID_X), device, torch.bfloat16)
    out["router_w"] = _randn((w.E, w.d), 1.0 / math.sqrt(w.d),
                             seed_for(awid, layer, _TID_RW), device, torch.float32)
    out["router_gamma"] = _randn((w.d,), 0.1, seed_for(awid, layer, _TID_GAMMA), device,
                                 torch.float32)
    out["router_bias"] = (zipf_bias(w.E, w.zipf_s, seed_for(w.wid, layer, _TID_BIAS), device)
                          if w.zipf_s > 0 else None)
    out["expert_gamma"] = (_randn((w.d,), 0.1, seed_for(w.wid, layer, _TID_EGAMMA), device,
                                  torch.float32) if w.expert_norm else None)
    if w.wdtype == WDTYPE_BF16:
        out["w_gate_up"] = _randn((w.E, 2 * w.f, w.d), 0.02, seed_for(w.wid, layer, _TID_WGU),
                                  device, torch.bfloat16)
        out["w_down"] = _randn((w.E, w.d, w.f), 0.02, seed_for(w.wid, layer, _TID_WD),
                               device, torch.bfloat16)
        out["scales_gate_up"] = None
        out["scales_down"] = None
    else:
        mk = {WDTYPE_FP8: make_fp8, WDTYPE_FP4: make_fp4}.get(w.wdtype, make_int4)
        out["w_gate_up"], out["scales_gate_up"] = mk(
            (w.E, 2 * w.f, w.d), seed_for(w.wid, layer, _TID_WGU),
            seed_for(w.wid, layer, _TID_SGU), device)
        out["w_down"], out["scales_down"] = mk(
            (w.E, w.d, w.f), seed_for(w.wid, layer, _TID_WD),
            seed_for(w.wid, layer, _TID_SD), device)
    return out


def make_small(T, d, E, k, f, seed, wdtype=WDTYPE_BF16, bias=False, residual=False,
               device="cpu", w_std=0.02, gamma_std=0.1, expert_norm=False) -> dict:
    """A small random layer of arbitrary shape for tests (same distributions)."""
    base = 100000 + 1000 * seed
    out = {
        "x": _randn((T, d), 1.0, base + 1, device, torch.bfloat16),
        "router_w": _randn((E, d), 1.0 / math.sqrt(d), base + 2, device, torch.float32),
        "router_gamma": _randn((d,), gamma_std, base + 3, device, torch.float32),
        "router_bias": _randn((E,), 1.0, base + 4, device, torch.float32) if bias else None,
        "residual": _randn((T, d), 1.0, base + 5, device, torch.bfloat16) if residual else None,
        "expert_gamma": (_randn((d,), gamma_std, base + 10, device, torch.float32)
                         if expert_norm else None),
    }
    if wdtype == WDTYPE_BF16:
        out["w_gate_up"] = _randn((E, 2 * f, d), w_std, base + 6, device, torch.bfloat16)
        out["w_down"] = _randn((E, d, f), w_std, base + 7, device, torch.bfloat16)
        out["scales_gate_up"] = None
        out["scales_down"] = None
    else:
        mk = {WDTYPE_FP8: make_fp8, WDTYPE_FP4: make_fp4}.get(wdtype, make_int4)
        out["w_gate_up"], out["scales_gate_up"] = mk((E, 2 * f, d), base + 6, base + 8, device)
        out["w_down"], out["scales_down"] = mk((E, d, f), base + 7, base + 9, device)
    return out


# ---------------------------------------------------------------- lm_head step
LMHEAD_V = 262144   # vocabulary of the lm_head (DiffusionGemma, vocab 262k)
LMHEAD_D = 2816


def make_lmhead(T: int, V: int, d: int, seed: int, device="cpu", logit_std: float = 2.0,
                max_boost: float = 30.0):
    """h [T, d] bf16 and W [V, d] bf16 for the lm_head step.  W ~ N(0,
    logit_std^2 / d), so a random h ~ N(0, 1) gives logits of std logit_std
    (a flat distribution); token t also gets c_t * W[v_t] / |W[v_t]|^2 added
    with c_t spread over [0, max_boost] and v_t random, so its logit of v_t
    is raised by about c_t and the entropies span flat to fully peaked, as
    a denoising canvas does."""
    g = _gen(seed, device)
    W = torch.randn((V, d), generator=g, device=device) * (logit_std / math.sqrt(d))
    h = torch.randn((T, d), generator=g, device=device)
    tgt = torch.randint(0, V, (T,), generator=g, device=device)
    c = torch.linspace(0.0, max_boost, T, device=device)[torch.randperm(T, generator=g, device=device)]
    wt = W[tgt]
    h += c[:, None] * wt / (wt * wt).sum(-1, keepdim=True)
    return h.to(torch.bfloat16), W.to(torch.bfloat16), tgt
