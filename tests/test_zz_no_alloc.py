"""moe_forward_noalloc: the layer for callers that cannot allocate device
memory (a host that pre-assigns all of the GPU's memory, or a loop that must
never enter the CUDA allocator).  Its intermediates live in the library's
fixed device array instead of a plan workspace.

Checked through the C ABI against moe_forward on the same inputs, on two
calls in a row (the array keeps the previous call's contents, so the second
call shows that what must start at zero is cleared).  Both paths run the same
kernels on the same bytes, so the outputs must be bit-identical.  The size
limit is enforced before anything is launched, and a device-side error of a
call made without a status pointer still reaches moe_plan_sync_status.  This
file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import block_diffusion_moe_router_b200 as moe
from block_diffusion_moe_router_b200 import _abi, inputs

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _call_noalloc(plan, T, lay, x, out, status, residual=None, bias=None):
    P = ctypes.c_void_p
    return _abi.lib().moe_forward_noalloc(
        P(plan), T, _ptr(x), _ptr(lay["router_w"]), _ptr(lay["router_gamma"]), _ptr(bias),
        None, _ptr(lay["w_gate_up"]), _ptr(lay["w_down"]), None, None, _ptr(residual),
        _ptr(out), _ptr(status), P(torch.cuda.current_stream().cuda_stream))


def _reference(plan, w, lay, x, residual=None, bias=None):
    ref = torch.empty((w.T, w.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(plan, w.T, x, lay["router_w"], lay["router_gamma"], bias, lay["w_gate_up"],
                    lay["w_down"], None, None, residual, ref)
    assert moe.moe_plan_sync_status(plan) == moe.MOE_OK
    return ref


def test_noalloc_matches_forward_on_two_calls():
    w = inputs.WORKLOADS["canvas"]
    lay = inputs.make_layer(w, device="cuda")
    x2 = inputs._randn((w.T, w.d), 1.0, 99123, "cuda", torch.bfloat16)
    plan = moe.moe_plan_create(w.E, w.k, w.d, w.f)
    try:
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        for x in (lay["x"], x2):
            ref = _reference(plan, w, lay, x)
            got = torch.full((w.T, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
            assert _call_noalloc(plan, w.T, lay, x, got, status) == moe.MOE_OK
            torch.cuda.synchronize()
            assert int(status.item()) == moe.MOE_OK
            assert torch.equal(got, ref)
    finally:
        moe.moe_plan_destroy(plan)


def test_noalloc_residual_and_router_bias():
    """A residual added in place (out aliases it) and a router bias that moves
    the expert choice: still the moe_forward bytes, on two calls in a row."""
    w = inputs.WORKLOADS["canvas"]
    lay = inputs.make_layer(w, device="cuda")
    bias = inputs.zipf_bias(w.E, 1.1, 4321, "cuda")
    res = inputs._randn((w.T, w.d), 1.0, 5151, "cuda", torch.bfloat16)
    plan = moe.moe_plan_create(w.E, w.k, w.d, w.f)
    try:
        for _ in range(2):
            ref = _reference(plan, w, lay, lay["x"], residual=res.clone(), bias=bias)
            buf = res.clone()
            assert _call_noalloc(plan, w.T, lay, lay["x"], buf, None, residual=buf,
                                 bias=bias) == moe.MOE_OK
            assert moe.moe_plan_sync_status(plan) == moe.MOE_OK
            assert torch.equal(buf, ref)
    finally:
        moe.moe_plan_destroy(plan)


def test_noalloc_error_reaches_sync_status_without_status_pointer():
    """The expert kernel's dependency wait is pointed at a flag nothing sets
    (bounded: it gives up after 20 ms).  With no status pointer given, the
    timeout is still reported by moe_plan_sync_status, and the next call is
    clean and correct."""
    T, E, k, d, f = 32, 16, 2, 256, 64
    lay = {key: (v.cuda() if isinstance(v, torch.Tensor) else v)
           for key, v in inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=2).items()}

    class W:
        pass

    w = W()
    w.T, w.d = T, d
    plan = moe.moe_plan_create(E, k, d, f)
    try:
        ref = _reference(plan, w, lay, lay["x"])
        moe.moe_plan_set_option(plan, moe.MOE_OPT_TIMEOUT_MS, 20)
        moe.moe_plan_set_option(plan, moe.MOE_OPT_TEST_STALL, 1)
        out = torch.empty_like(ref)
        assert _call_noalloc(plan, T, lay, lay["x"], out, None) == moe.MOE_OK
        assert moe.moe_plan_sync_status(plan) == moe.MOE_ERR_TIMEOUT
        assert moe.moe_plan_sync_status(plan) == moe.MOE_OK  # read once, then cleared
        moe.moe_plan_set_option(plan, moe.MOE_OPT_TEST_STALL, 0)
        assert _call_noalloc(plan, T, lay, lay["x"], out, None) == moe.MOE_OK
        assert moe.moe_plan_sync_status(plan) == moe.MOE_OK
        assert torch.equal(out, ref)
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
