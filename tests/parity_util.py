"""Shared checks for the GPU-vs-oracle parity tests.

Acceptance (floating point): relative L2 error of the layer output against
the fp64 oracle <= 5e-3 for bf16 weights (1e-2 for int4), over the whole
[T, d] tensor.  fp8 (E4M3) weights take the bf16 bound: their values reach
the tensor cores exactly (every E4M3 value is an fp16 value), the
activations are fp16 (bf16 inputs convert exactly; h is rounded once, to 11
significant bits instead of bf16's 8) and the row scale is applied to the
fp32 accumulator, so no step rounds more coarsely than on the bf16 path.  Integer work is bit-exact: expert indices on every token
whose oracle gap z_(k) - z_(k+1) is at least 1e-5, and the routing tables.
A token below that gap is "flagged": its GPU set must be one of the sets the
oracle's own logits allow, and its output is compared with the oracle run on
that set.
"""
from __future__ import annotations

import numpy as np

import oracle

GAP_FLAG = 1e-5
TOL_BF16 = 5e-3
TOL_INT4 = 1e-2
TOL_FP8 = TOL_BF16
TOL_FP4 = TOL_BF16  # exact block-scaled decode; fp16 activations as on the fp8 path


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def valid_alternative(gpu_set, z_row, k) -> bool:
    """gpu_set is a valid top-k under a near-tie of the oracle logits."""
    order = sorted(range(len(z_row)), key=lambda e: (-z_row[e], e))
    zk = z_row[order[k - 1]]
    must = {e for e in range(len(z_row)) if z_row[e] > zk + GAP_FLAG}
    allowed = {e for e in range(len(z_row)) if z_row[e] >= zk - GAP_FLAG}
    s = set(int(e) for e in gpu_set)
    return len(s) == k and must <= s <= allowed


def check_routing(gidx, gw, oidx, ow, ogap, z, k):
    """Indices exact on unflagged tokens, valid alternatives on flagged ones,
    weights close where the sets agree.  Returns the mismatching rows."""
    gidx = np.asarray(gidx)
    mism = np.nonzero((gidx != oidx).any(axis=1))[0]
    for t in mism:
        assert ogap[t] < GAP_FLAG, f"token {t}: GPU {gidx[t]} vs oracle {oidx[t]}, gap {ogap[t]}"
        assert valid_alternative(gidx[t], z[t], k), f"token {t}: invalid alternative set"
    ok = np.ones(len(gidx), bool)
    ok[mism] = False
    np.testing.assert_allclose(np.asarray(gw)[ok], ow[ok], rtol=1e-4, atol=1e-6)
    return mism


def oracle_rows_for_sets(lay, k, rows, sets, eps=1e-6):
    """Oracle output of the given token rows with their selected sets ordered
    by the oracle's own logits (used only for flagged tokens)."""
    sub = {key: (v[rows] if key in ("x", "residual") and v is not None else v)
           for key, v in lay.items()}
    _, _, _, z = oracle.route(sub["x"], sub["router_w"], sub["router_gamma"],
                              sub.get("router_bias"), k, eps=eps)
    forced = np.array([sorted(list(s), key=lambda e: (-z[i][e], e)) for i, s in enumerate(sets)],
                      np.int32)
    out, _, _, _ = oracle.moe_forward(sub["x"], sub["router_w"], sub["router_gamma"],
                                      sub.get("router_bias"), sub["w_gate_up"], sub["w_down"], k,
                                      scales_gate_up=sub.get("scales_gate_up"),
                                      scales_down=sub.get("scales_down"),
                                      residual=sub.get("residual"), forced_idx=forced, eps=eps,
                                      expert_gamma=sub.get("expert_gamma"))
    return out


def stable_tables(idx, E):
    """Expected routing tables from top-k indices: a stable counting sort of
    the assignments a = t*k + j by expert."""
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")        # slot -> assignment
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm = (order // k).astype(np.int32)
    slot_of = np.empty_like(order)
    slot_of[order] = np.arange(len(order))
    return offsets, perm, slot_of.astype(np.int32)
