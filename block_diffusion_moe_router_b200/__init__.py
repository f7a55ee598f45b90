"""B200-native (sm_100a) top-k mixture-of-experts FFN layer, DiffusionGemma
26B-A4B shape: hidden 2816, 128 experts, top-8, per-expert intermediate 704,
GELU-tanh gated experts, router with its own (1+gamma) RMSNorm.

The C ABI (include/moe.h) lives in libmoe_b200.so; `_abi` binds it with the
same function names.  `MoeLayer` is a small convenience wrapper over a plan.
Importing this package does not load the library; the first call does, and
fails loudly if it has not been built.
"""
from __future__ import annotations

from . import _abi
from ._abi import (  # noqa: F401
    MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_ALLOC, MOE_ERR_CUDA,
    MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_CHECK, MOE_W_BF16, MOE_W_INT4_G128, MOE_W_FP8_E4M3, MOE_W_FP4_E2M1, MOE_OPT_EPS,
    MOE_OPT_TIMEOUT_MS, MOE_OPT_PROFILE, MOE_OPT_TEST_STALL, MOE_OPT_PDL,
    MOE_OPT_L2_PREFETCH_MB, MOE_OPT_ROUTER, MOE_OPT_Y_BF16, MOE_OPT_DEBUG, MOE_OPT_CHUNK_TOKENS, MOE_MAX_T,
    MOE_MAX_ASSIGNMENTS, MOE_K_ROUTER, MOE_K_PLAN,
    MOE_K_EXPERT, MOE_K_COMBINE, KERNEL_NAMES, MoeError,
    moe_plan_create, moe_plan_set_option, moe_plan_reserve, moe_forward, moe_forward_host,
    moe_forward_noalloc,
    moe_route, moe_plan_routing, moe_plan_sync_status, moe_plan_profile, moe_plan_destroy,
    moe_status_str, moe_lmhead_create, moe_lmhead_forward, moe_lmhead_sync_status,
    moe_lmhead_destroy, moe_lmhead_set_profile, moe_lmhead_profile, moe_ep_dispatch,
    moe_expert_rows, moe_combine_rows,
)


class MoeLayer:
    """Owns one plan.  Tensors are torch CUDA tensors laid out as in moe.h."""

    def __init__(self, E: int, k: int, d: int, f: int, wdtype: int = MOE_W_BF16):
        self.E, self.k, self.d, self.f, self.wdtype = E, k, d, f, wdtype
        self.plan = moe_plan_create(E, k, d, f, wdtype)

    def close(self):
        if self.plan:
            moe_plan_destroy(self.plan)
            self.plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, x, router_w, router_gamma, w_gate_up, w_down, router_bias=None,
                scales_gate_up=None, scales_down=None, residual=None, out=None, stream=None,
                expert_gamma=None):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.d), dtype=torch.bfloat16, device=x.device)
        moe_forward(self.plan, T, x, router_w, router_gamma, router_bias, w_gate_up, w_down,
                    scales_gate_up, scales_down, residual, out, stream,
                    expert_gamma=expert_gamma)
        return out

    def route(self, x, router_w, router_gamma, router_bias=None, stream=None):
        import torch
        T = x.shape[0]
        idx = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        gap = torch.empty((T,), dtype=torch.float32, device=x.device)
        moe_route(self.plan, T, x, router_w, router_gamma, router_bias, idx, w, gap, stream)
        return idx, w, gap

    def routing_tables(self, T: int, stream=None):
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        off = torch.empty(self.E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * self.k, dtype=torch.int32, device=dev)
        slot_of = torch.empty(T * self.k, dtype=torch.int32, device=dev)
        moe_plan_routing(self.plan, off, perm, slot_of, stream)
        return off, perm, slot_of

    def sync_status(self, stream=None) -> int:
        return moe_plan_sync_status(self.plan, stream)


class LmHead:
    """lm_head over the canvas plus the entropy-bound acceptance step (a thin
    owner of an moe_lmhead_t; every step runs in the library's kernels)."""

    def __init__(self, V: int, d: int):
        self.V, self.d = V, d
        self.handle = moe_lmhead_create(V, d)

    def step(self, h, w, temperature=1.0, softcap=0.0, masked=None, entropy_bound=0.1,
             stream=None):
        import torch
        T = h.shape[0]
        dev = h.device
        token = torch.empty(T, dtype=torch.int32, device=dev)
        ent = torch.empty(T, dtype=torch.float32, device=dev)
        logz = torch.empty(T, dtype=torch.float32, device=dev)
        acc = torch.empty(T, dtype=torch.uint8, device=dev)
        moe_lmhead_forward(self.handle, T, h, w, temperature, softcap, masked, entropy_bound,
                           token, ent, logz, acc, stream)
        return token, ent, logz, acc

    def sync_status(self, stream=None) -> int:
        return moe_lmhead_sync_status(self.handle, stream)

    def close(self):
        if self.handle:
            moe_lmhead_destroy(self.handle)
            self.handle = None
