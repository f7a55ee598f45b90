"""moe_forward_noalloc: the layer for callers that cannot allocate device
memory (a host that pre-assigns all of the GPU's memory, or a loop that must
never enter the CUDA allocator).  Its intermediates live in the library's
fixed device array instead of a plan workspace.

Checked through the C ABI against moe_forward on the same inputs, on two
calls in a row (the array keeps the previous call's contents, so the second
call shows that what must start at zero is cleared), with the same rel-L2
tolerance as the oracle parity tests; and the size limit is enforced before
anything is launched.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_diffusion_moe_router_b200 as moe
from block_diffusion_moe_router_b200 import _abi, inputs

pytestmark = pytest.mark.gpu

TOL = 5e-3  # the bf16 tolerance of the parity tests


def _rel(a, b):
    a = a.double()
    b = b.double()
    return float((a - b).norm() / b.norm())


def _call_noalloc(plan, T, lay, x, out, status):
    P = ctypes.c_void_p
    return _abi.lib().moe_forward_noalloc(
        P(plan), T, P(x.data_ptr()), P(lay["router_w"].data_ptr()),
        P(lay["router_gamma"].data_ptr()), None, None, P(lay["w_gate_up"].data_ptr()),
        P(lay["w_down"].data_ptr()), None, None, None, P(out.data_ptr()),
        P(status.data_ptr()), P(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_forward_on_two_calls():
    w = inputs.WORKLOADS["canvas"]
    lay = inputs.make_layer(w, device="cuda")
    x2 = inputs._randn((w.T, w.d), 1.0, 99123, "cuda", torch.bfloat16)
    plan = moe.moe_plan_create(w.E, w.k, w.d, w.f)
    try:
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        for x in (lay["x"], x2):
            ref = torch.empty((w.T, w.d), dtype=torch.bfloat16, device="cuda")
            moe.moe_forward(plan, w.T, x, lay["router_w"], lay["router_gamma"], None,
                            lay["w_gate_up"], lay["w_down"], None, None, None, ref)
            assert moe.moe_plan_sync_status(plan) == moe.MOE_OK
            got = torch.full((w.T, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
            assert _call_noalloc(plan, w.T, lay, x, got, status) == moe.MOE_OK
            torch.cuda.synchronize()
            assert int(status.item()) == moe.MOE_OK
            assert torch.isfinite(got.float()).all()
            err = _rel(got.float(), ref.float())
            assert err <= TOL, err
            print("noalloc vs forward rel-L2", err, "bitwise", torch.equal(got, ref))
    finally:
        moe.moe_plan_destroy(plan)


def test_noalloc_rejects_calls_beyond_the_array():
    w = inputs.WORKLOADS["canvas"]
    plan = moe.moe_plan_create(w.E, w.k, w.d, w.f)
    try:
        T = 1024  # 4 canvases: about 150 MB of intermediates > 40 MiB
        lay = inputs.make_layer(w, device="cuda", T=T)
        out = torch.zeros((T, w.d), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros((1,), dtype=torch.int32, device="cuda")
        assert _call_noalloc(plan, T, lay, lay["x"], out, status) == moe.MOE_ERR_UNSUPPORTED
        torch.cuda.synchronize()
        assert torch.count_nonzero(out) == 0  # nothing was launched
    finally:
        moe.moe_plan_destroy(plan)
