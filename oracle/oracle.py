"""ctypes binding of moe_oracle.c (built with gcc into oracle/_build/).

TEST INFRASTRUCTURE ONLY (tests, smoke check, bench CPU baseline).
All array arguments are torch CPU tensors or numpy arrays; results come back
as numpy arrays (float64 / int32).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

W_BF16 = 0
W_INT4 = 1
W_FP8 = 2
W_FP4 = 3


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (-O2, OpenMP, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _SO)
    return _SO


_SRC32 = os.path.join(_HERE, "moe_oracle_f32.c")
_SO32 = os.path.join(_BUILD, "liboracle_f32.so")
_lib32 = None


def build_f32(force: bool = False) -> str:
    """Compile the single-precision timing build (moe_oracle_f32.c, which
    includes moe_oracle.c with every double made a float)."""
    os.makedirs(_BUILD, exist_ok=True)
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC32))
    if force or not os.path.exists(_SO32) or os.path.getmtime(_SO32) < newest:
        tmp = _SO32 + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-Wall", "-o", tmp, _SRC32, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _SO32)
    return _SO32


def lib_f32():
    """The timing build: the same entry points with float arguments."""
    global _lib32
    with _lock:
        if _lib32 is None:
            build_f32()
            L = ctypes.CDLL(_SO32)
            P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            L.oracle_moe_forward.argtypes = [I, I, I, I, I, I, P, P, P, P, P, F, P, P, P, P, P,
                                             P, P, P, P, P]
            L.oracle_set_threads.argtypes = [I]
            L.oracle_get_threads.restype = I
            _lib32 = L
    return _lib32


def moe_forward_f32(x, router_w, router_gamma, router_bias, w_gate_up, w_down, k: int,
                    scales_gate_up=None, scales_down=None, residual=None, eps: float = 1e-6,
                    expert_gamma=None):
    """The whole layer in single precision (timing build): out [T,d] float32."""
    x = _np(x)
    rw = _np(router_w, np.float32)
    g = _np(router_gamma, np.float32)
    b = _np(router_bias, np.float32)
    wgu = _np(w_gate_up)
    wd = _np(w_down)
    sgu = _np(scales_gate_up)
    sd = _np(scales_down)
    res = _np(residual)
    eg = _np(expert_gamma, np.float32)
    T, d = x.shape
    E = rw.shape[0]
    out = np.empty((T, d), np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    gap = np.empty(T, np.float32)
    lib_f32().oracle_moe_forward(T, E, k, d, wgu.shape[1] // 2, _wdtype(wgu, sgu), _p(x), _p(rw),
                                 _p(g), _p(b), _p(eg), float(eps), _p(wgu), _p(wd), _p(sgu),
                                 _p(sd), _p(res), None, _p(out), _p(idx), _p(w), _p(gap))
    return out


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            P = ctypes.c_void_p
            I = ctypes.c_int
            D = ctypes.c_double
            L.oracle_gelu_tanh.restype = D
            L.oracle_gelu_tanh.argtypes = [D]
            L.oracle_gelu_tanh_vec.argtypes = [I, P, P]
            L.oracle_rmsnorm_rows.argtypes = [I, I, P, P, D, P]
            L.oracle_select_topk.argtypes = [I, I, P, P, P]
            L.oracle_route_weights.argtypes = [I, I, P, P, P]
            L.oracle_route.argtypes = [I, I, I, I, P, P, P, P, D, P, P, P, P]
            L.oracle_moe_forward.argtypes = [I, I, I, I, I, I, P, P, P, P, P, D, P, P, P, P, P,
                                             P, P, P, P, P]
            L.oracle_expert_ffn.argtypes = [I, I, I, P, P, P, P, I, P, P, P]
            L.oracle_weight_row.argtypes = [I, P, P, I, I, I, I, P]
            L.oracle_decode_bf16.argtypes = [I, P, P]
            L.oracle_decode_fp16.argtypes = [I, P, P]
            L.oracle_decode_e4m3.argtypes = [I, P, P]
            L.oracle_decode_e2m1.argtypes = [I, P, P]
            L.oracle_lmhead_stats.argtypes = [I, I, P, P, D, D, P, I, P, P, P, P]
            L.oracle_eb_accept.argtypes = [I, P, P, D, P]
            L.oracle_set_threads.argtypes = [I]
            L.oracle_get_threads.restype = I
            _lib = L
    return _lib


def _np(t, dtype=None):
    """Contiguous numpy view of a torch CPU tensor / numpy array (bf16 and
    fp16 tensors are viewed as raw uint16 bits)."""
    if t is None:
        return None
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().cpu().contiguous()
            if t.dtype in (torch.bfloat16, torch.float16):
                t = t.view(torch.int16)
            a = t.numpy()
            if a.dtype == np.int16:
                a = a.view(np.uint16)
            t = a
    except ImportError:
        pass
    a = np.ascontiguousarray(t)
    if dtype is not None and a.dtype != dtype:
        a = a.astype(dtype)
    return a


def _wdtype(w, scales) -> int:
    """Storage format of a weight array: bf16 (uint16 bits), int4 (packed
    bytes with fp16 scales), fp8 E4M3 (one byte per weight, fp32 row
    scales) or fp4 E2M1 (packed bytes, scale records as uint8 bytes)."""
    if w.dtype != np.uint8:
        return W_BF16
    if scales is not None and scales.dtype == np.float32:
        return W_FP8
    if scales is not None and scales.dtype == np.uint8:
        return W_FP4
    return W_INT4


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


def gelu_tanh(a) -> np.ndarray:
    a = _np(a, np.float64)
    out = np.empty_like(a)
    lib().oracle_gelu_tanh_vec(a.size, _p(a), _p(out))
    return out


def rmsnorm_plus_one(x, gamma, eps: float) -> np.ndarray:
    """x [T,d] float64, gamma [d] float32 -> u [T,d]."""
    x = _np(x, np.float64)
    gamma = _np(gamma, np.float32)
    T, d = x.shape
    out = np.empty_like(x)
    lib().oracle_rmsnorm_rows(T, d, _p(x), _p(gamma), float(eps), _p(out))
    return out


def select_topk(z, k: int):
    """z [E] float64 -> (idx [k] int32, gap float)."""
    z = _np(z, np.float64)
    idx = np.empty(k, np.int32)
    gap = np.zeros(1, np.float64)
    lib().oracle_select_topk(z.size, k, _p(z), _p(idx), _p(gap))
    return idx, float(gap[0])


def route_weights(z, idx) -> np.ndarray:
    z = _np(z, np.float64)
    idx = _np(idx, np.int32)
    w = np.empty(idx.size, np.float64)
    lib().oracle_route_weights(z.size, idx.size, _p(z), _p(idx), _p(w))
    return w


def route(x, router_w, router_gamma, router_bias, k: int, eps: float = 1e-6):
    """Routing of every token: (idx [T,k] int32, w [T,k], gap [T], z [T,E])."""
    x = _np(x)
    rw = _np(router_w, np.float32)
    g = _np(router_gamma, np.float32)
    b = _np(router_bias, np.float32)
    T, d = x.shape
    E = rw.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    gap = np.empty(T, np.float64)
    z = np.empty((T, E), np.float64)
    lib().oracle_route(T, E, k, d, _p(x), _p(rw), _p(g), _p(b), float(eps), _p(idx), _p(w),
                       _p(gap), _p(z))
    return idx, w, gap, z


def moe_forward(x, router_w, router_gamma, router_bias, w_gate_up, w_down, k: int,
                scales_gate_up=None, scales_down=None, residual=None, forced_idx=None,
                eps: float = 1e-6, expert_gamma=None):
    """The whole layer: (out [T,d] float64, idx [T,k], w [T,k], gap [T]).
    expert_gamma (or None): the experts read rmsnorm(x) * (1 + expert_gamma)."""
    x = _np(x)
    rw = _np(router_w, np.float32)
    g = _np(router_gamma, np.float32)
    b = _np(router_bias, np.float32)
    wgu = _np(w_gate_up)
    wd = _np(w_down)
    sgu = _np(scales_gate_up)
    sd = _np(scales_down)
    res = _np(residual)
    fi = _np(forced_idx, np.int32)
    eg = _np(expert_gamma, np.float32)
    T, d = x.shape
    E = rw.shape[0]
    wdtype = _wdtype(wgu, sgu)
    f = wgu.shape[1] // 2
    assert wgu.shape[0] == E and wd.shape[0] == E
    if wdtype != W_BF16:
        assert sgu is not None and sd is not None
    out = np.empty((T, d), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    gap = np.empty(T, np.float64)
    lib().oracle_moe_forward(T, E, k, d, f, wdtype, _p(x), _p(rw), _p(g), _p(b), _p(eg),
                             float(eps), _p(wgu), _p(wd), _p(sgu), _p(sd), _p(res), _p(fi),
                             _p(out), _p(idx), _p(w), _p(gap))
    return out, idx, w, gap


def expert_ffn(x_row, e: int, w_gate_up, w_down, scales_gate_up=None, scales_down=None):
    """One expert on one token row (float64 [d]) -> (y [d], h [f])."""
    x_row = _np(x_row, np.float64)
    wgu = _np(w_gate_up)
    wd = _np(w_down)
    sgu = _np(scales_gate_up)
    sd = _np(scales_down)
    d = x_row.size
    f = wgu.shape[1] // 2
    wdtype = _wdtype(wgu, sgu)
    y = np.empty(d, np.float64)
    h = np.empty(f, np.float64)
    lib().oracle_expert_ffn(d, f, wdtype, _p(wgu), _p(wd), _p(sgu), _p(sd), int(e), _p(x_row),
                            _p(y), _p(h))
    return y, h


def weight_row(w, scales, e: int, r: int, cols: int) -> np.ndarray:
    """Row r of expert e of a [E,R,C] weight, widened / dequantised to fp64."""
    w = _np(w)
    s = _np(scales)
    wdtype = _wdtype(w, s)
    R = w.shape[1]
    out = np.empty(cols, np.float64)
    lib().oracle_weight_row(wdtype, _p(w), _p(s), R, cols, int(e), int(r), _p(out))
    return out


def decode_bf16(t) -> np.ndarray:
    a = _np(t)
    out = np.empty(a.shape, np.float64)
    lib().oracle_decode_bf16(a.size, _p(a), _p(out))
    return out


def decode_fp16(t) -> np.ndarray:
    a = _np(t)
    out = np.empty(a.shape, np.float64)
    lib().oracle_decode_fp16(a.size, _p(a), _p(out))
    return out


def decode_e2m1(t) -> np.ndarray:
    """E2M1 codes (the low nibble of each uint8) -> float64 values."""
    a = _np(t, np.uint8)
    out = np.empty(a.shape, np.float64)
    lib().oracle_decode_e2m1(a.size, _p(a), _p(out))
    return out


def decode_e4m3(t) -> np.ndarray:
    """E4M3 bytes (uint8) -> float64 values (NaN for the NaN codes)."""
    a = _np(t, np.uint8)
    out = np.empty(a.shape, np.float64)
    lib().oracle_decode_e4m3(a.size, _p(a), _p(out))
    return out


def lmhead_stats(h, W, rows=None, temperature: float = 1.0, softcap: float = 0.0):
    """Per token row of h [T,d] (bf16) against the lm_head W [V,d] (bf16):
    (logZ, entropy H, argmax, gap between the two largest scaled logits),
    all of softmax(z / temperature) with z = h . W (soft-capped if softcap > 0)."""
    h = _np(h)
    W = _np(W)
    T, d = h.shape
    V = W.shape[0]
    rows = np.arange(T, dtype=np.int32) if rows is None else np.asarray(rows, np.int32)
    n = rows.size
    logz = np.empty(n, np.float64)
    H = np.empty(n, np.float64)
    am = np.empty(n, np.int32)
    gap = np.empty(n, np.float64)
    lib().oracle_lmhead_stats(V, d, _p(h), _p(W), 1.0 / temperature, float(softcap), _p(rows), n,
                              _p(logz), _p(H), _p(am), _p(gap))
    return logz, H, am, gap


def eb_accept(H, masked, bound: float) -> np.ndarray:
    """Entropy-bounded acceptance (uint8 per position) over the masked ones."""
    H = _np(H, np.float64)
    T = H.size
    m = None if masked is None else _np(masked, np.uint8)
    acc = np.empty(T, np.uint8)
    lib().oracle_eb_accept(T, _p(H), _p(m), float(bound), _p(acc))
    return acc
