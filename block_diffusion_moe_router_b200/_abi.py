"""ctypes binding of libmoe_b200.so (declared in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensor arguments may be torch tensors (their data_ptr() is
passed) or raw integer addresses.  There is no fallback: if the library is
missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_ALLOC = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_DEVICE_CHECK = 6

MOE_W_BF16 = 0
MOE_W_INT4_G128 = 1
MOE_W_FP8_E4M3 = 2
MOE_W_FP4_E2M1 = 3

MOE_OPT_EPS = 0
MOE_OPT_TIMEOUT_MS = 1
MOE_OPT_PROFILE = 2
MOE_OPT_TEST_STALL = 3
MOE_OPT_PDL = 4
MOE_OPT_L2_PREFETCH_MB = 5
MOE_OPT_ROUTER = 6
MOE_OPT_Y_BF16 = 7
MOE_OPT_DEBUG = 8
MOE_OPT_CHUNK_TOKENS = 9

MOE_MAX_T = 65536
MOE_MAX_ASSIGNMENTS = 1 << 19

MOE_K_ROUTER, MOE_K_PLAN, MOE_K_EXPERT, MOE_K_COMBINE = range(4)
KERNEL_NAMES = ["router", "plan_gather", "expert", "combine"]

# Every function include/moe.h declares.
EXPORTS = [
    "moe_plan_create", "moe_plan_set_option", "moe_plan_reserve", "moe_forward",
    "moe_forward_host", "moe_route", "moe_plan_routing", "moe_plan_sync_status",
    "moe_plan_profile", "moe_plan_destroy", "moe_status_str", "moe_forward_noalloc",
    "moe_lmhead_create", "moe_lmhead_forward", "moe_lmhead_sync_status", "moe_lmhead_destroy",
    "moe_lmhead_set_profile", "moe_lmhead_profile", "moe_ep_dispatch", "moe_expert_rows",
    "moe_combine_rows",
]

_lock = threading.Lock()
_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)}")


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is not built; run `python -c 'import __graft_entry__ as g; "
                    f"g.build()'` (there is no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
            L.moe_plan_create.argtypes = [I, I, I, I, I, ctypes.POINTER(P)]
            L.moe_plan_create.restype = I
            L.moe_plan_set_option.argtypes = [P, I, D]
            L.moe_plan_set_option.restype = I
            L.moe_plan_reserve.argtypes = [P, I]
            L.moe_plan_reserve.restype = I
            L.moe_forward.argtypes = [P, I, P, P, P, P, P, P, P, P, P, P, P, P]
            L.moe_forward.restype = I
            L.moe_forward_host.argtypes = [P, I, P, P, P, P, P, P, P, P, P, P, P, P]
            L.moe_forward_host.restype = I
            L.moe_route.argtypes = [P, I, P, P, P, P, P, P, P, P]
            L.moe_route.restype = I
            L.moe_plan_routing.argtypes = [P, P, P, P, P]
            L.moe_plan_routing.restype = I
            L.moe_plan_sync_status.argtypes = [P, P]
            L.moe_plan_sync_status.restype = I
            L.moe_plan_profile.argtypes = [P, I, ctypes.POINTER(D), ctypes.POINTER(I)]
            L.moe_plan_profile.restype = I
            L.moe_plan_destroy.argtypes = [P]
            L.moe_plan_destroy.restype = None
            L.moe_forward_noalloc.argtypes = [P, I, P, P, P, P, P, P, P, P, P, P, P, P, P]
            L.moe_forward_noalloc.restype = I
            L.moe_ep_dispatch.argtypes = [P, I, P, P, I, P, P, P, P, P, P]
            L.moe_ep_dispatch.restype = I
            L.moe_expert_rows.argtypes = [P, I, P, P, P, P, P, P, P, P, P]
            L.moe_expert_rows.restype = I
            L.moe_combine_rows.argtypes = [P, I, P, P, P, P, P, P]
            L.moe_combine_rows.restype = I
            L.moe_status_str.argtypes = [I]
            L.moe_status_str.restype = ctypes.c_char_p
            F = ctypes.c_float
            L.moe_lmhead_create.argtypes = [I, I, ctypes.POINTER(P)]
            L.moe_lmhead_create.restype = I
            L.moe_lmhead_forward.argtypes = [P, I, P, P, F, F, P, F, P, P, P, P, P]
            L.moe_lmhead_forward.restype = I
            L.moe_lmhead_sync_status.argtypes = [P, P]
            L.moe_lmhead_sync_status.restype = I
            L.moe_lmhead_destroy.argtypes = [P]
            L.moe_lmhead_destroy.restype = None
            L.moe_lmhead_set_profile.argtypes = [P, I]
            L.moe_lmhead_set_profile.restype = I
            L.moe_lmhead_profile.argtypes = [P, ctypes.POINTER(D), ctypes.POINTER(I)]
            L.moe_lmhead_profile.restype = I
            _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().moe_status_str(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        if not t.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return t.data_ptr()
    if hasattr(t, "ctypes"):  # numpy array (host memory)
        return t.ctypes.data
    raise TypeError(f"cannot pass {type(t)} as a pointer")


def _stream(s):
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, what: str, check: bool):
    if check and st != MOE_OK:
        raise MoeError(st, what)
    return st


def moe_plan_create(E: int, k: int, d: int, f: int, wdtype: int = MOE_W_BF16) -> int:
    h = ctypes.c_void_p()
    _check(lib().moe_plan_create(E, k, d, f, wdtype, ctypes.byref(h)), "moe_plan_create", True)
    return h.value


def moe_plan_set_option(plan: int, key: int, value: float, check: bool = True) -> int:
    return _check(lib().moe_plan_set_option(plan, key, float(value)), "moe_plan_set_option", check)


def moe_plan_reserve(plan: int, max_T: int, check: bool = True) -> int:
    return _check(lib().moe_plan_reserve(plan, max_T), "moe_plan_reserve", check)


def moe_forward(plan, T, x, router_w, router_gamma, router_bias, w_gate_up, w_down,
                scales_gate_up, scales_down, residual, out, stream=None, check: bool = True,
                expert_gamma=None):
    st = lib().moe_forward(plan, T, _ptr(x), _ptr(router_w), _ptr(router_gamma),
                           _ptr(router_bias), _ptr(expert_gamma), _ptr(w_gate_up), _ptr(w_down),
                           _ptr(scales_gate_up), _ptr(scales_down), _ptr(residual), _ptr(out),
                           _stream(stream))
    return _check(st, "moe_forward", check)


def moe_forward_host(plan, T, x_host, router_w, router_gamma, router_bias, w_gate_up, w_down,
                     scales_gate_up, scales_down, residual_host, out_host, stream=None,
                     check: bool = True, expert_gamma=None):
    st = lib().moe_forward_host(plan, T, _ptr(x_host), _ptr(router_w), _ptr(router_gamma),
                                _ptr(router_bias), _ptr(expert_gamma), _ptr(w_gate_up),
                                _ptr(w_down),
                                _ptr(scales_gate_up), _ptr(scales_down), _ptr(residual_host),
                                _ptr(out_host), _stream(stream))
    return _check(st, "moe_forward_host", check)


def moe_forward_noalloc(plan, T, x, router_w, router_gamma, router_bias, w_gate_up, w_down,
                        scales_gate_up, scales_down, residual, out, status_out=None, stream=None,
                        check: bool = True, expert_gamma=None):
    """moe_forward without any device allocation: intermediates live in the
    library's fixed 40 MiB device array (see include/moe.h)."""
    st = lib().moe_forward_noalloc(plan, T, _ptr(x), _ptr(router_w), _ptr(router_gamma),
                                   _ptr(router_bias), _ptr(expert_gamma), _ptr(w_gate_up),
                                   _ptr(w_down),
                                   _ptr(scales_gate_up), _ptr(scales_down), _ptr(residual),
                                   _ptr(out), _ptr(status_out), _stream(stream))
    return _check(st, "moe_forward_noalloc", check)


def moe_ep_dispatch(plan, T, x, idx, n_ranks, expert_gamma, send_rows, send_expert, pos,
                    send_counts, stream=None, check: bool = True):
    st = lib().moe_ep_dispatch(plan, T, _ptr(x), _ptr(idx), n_ranks, _ptr(expert_gamma),
                               _ptr(send_rows), _ptr(send_expert), _ptr(pos), _ptr(send_counts),
                               _stream(stream))
    return _check(st, "moe_ep_dispatch", check)


def moe_expert_rows(plan, R, x_rows, row_expert, expert_gamma, w_gate_up, w_down, scales_gate_up,
                    scales_down, y_rows, stream=None, check: bool = True):
    st = lib().moe_expert_rows(plan, R, _ptr(x_rows), _ptr(row_expert), _ptr(expert_gamma),
                               _ptr(w_gate_up), _ptr(w_down), _ptr(scales_gate_up),
                               _ptr(scales_down), _ptr(y_rows), _stream(stream))
    return _check(st, "moe_expert_rows", check)


def moe_combine_rows(plan, T, y_rows, pos, w, residual, out, stream=None, check: bool = True):
    st = lib().moe_combine_rows(plan, T, _ptr(y_rows), _ptr(pos), _ptr(w), _ptr(residual),
                                _ptr(out), _stream(stream))
    return _check(st, "moe_combine_rows", check)


def moe_route(plan, T, x, router_w, router_gamma, router_bias, idx_out, w_out, gap_out,
              stream=None, check: bool = True):
    st = lib().moe_route(plan, T, _ptr(x), _ptr(router_w), _ptr(router_gamma),
                         _ptr(router_bias), _ptr(idx_out), _ptr(w_out), _ptr(gap_out),
                         _stream(stream))
    return _check(st, "moe_route", check)


def moe_plan_routing(plan, offsets, perm, slot_of, stream=None, check: bool = True):
    st = lib().moe_plan_routing(plan, _ptr(offsets), _ptr(perm), _ptr(slot_of), _stream(stream))
    return _check(st, "moe_plan_routing", check)


def moe_plan_sync_status(plan, stream=None) -> int:
    return lib().moe_plan_sync_status(plan, _stream(stream))


def moe_plan_profile(plan, kernel: int):
    ms = ctypes.c_double()
    n = ctypes.c_int()
    _check(lib().moe_plan_profile(plan, kernel, ctypes.byref(ms), ctypes.byref(n)),
           "moe_plan_profile", True)
    return ms.value, n.value


def moe_plan_destroy(plan) -> None:
    if plan:
        lib().moe_plan_destroy(plan)


def moe_status_str(status: int) -> str:
    return status_str(status)


def moe_lmhead_create(V: int, d: int) -> int:
    h = ctypes.c_void_p()
    _check(lib().moe_lmhead_create(V, d, ctypes.byref(h)), "moe_lmhead_create", True)
    return h.value


def moe_lmhead_forward(lh, T, h, w, temperature, softcap, masked, entropy_bound, token_out,
                       entropy_out, logz_out, accept_out, stream=None, check: bool = True):
    st = lib().moe_lmhead_forward(lh, T, _ptr(h), _ptr(w), float(temperature), float(softcap),
                                  _ptr(masked), float(entropy_bound), _ptr(token_out),
                                  _ptr(entropy_out), _ptr(logz_out), _ptr(accept_out),
                                  _stream(stream))
    return _check(st, "moe_lmhead_forward", check)


def moe_lmhead_sync_status(lh, stream=None) -> int:
    return lib().moe_lmhead_sync_status(lh, _stream(stream))


def moe_lmhead_destroy(lh) -> None:
    lib().moe_lmhead_destroy(lh)


def moe_lmhead_set_profile(lh, on: bool) -> None:
    _check(lib().moe_lmhead_set_profile(lh, 1 if on else 0), "moe_lmhead_set_profile", True)


def moe_lmhead_profile(lh):
    """(total GEMM ms, launches) recorded since the last read."""
    ms = ctypes.c_double()
    n = ctypes.c_int()
    _check(lib().moe_lmhead_profile(lh, ctypes.byref(ms), ctypes.byref(n)), "moe_lmhead_profile",
           True)
    return ms.value, n.value
