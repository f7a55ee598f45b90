"""Pins of the oracle's lm_head statistics and entropy-bounded acceptance
against library routines (torch logsumexp / softmax / argmax / tanh), closed
forms and a brute-force restatement of the acceptance rule."""
import math

import numpy as np
import pytest
import torch

import oracle


def _case(T, V, d, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn(T, d, generator=g).to(torch.bfloat16)
    W = (torch.randn(V, d, generator=g) * scale / math.sqrt(d)).to(torch.bfloat16)
    return h, W


@pytest.mark.parametrize("temperature,softcap", [(1.0, 0.0), (0.8, 0.0), (0.4, 30.0), (0.6, 2.0)])
def test_stats_match_torch(temperature, softcap):
    h, W = _case(T=7, V=300, d=96, seed=1, scale=4.0)
    logz, H, am, gap = oracle.lmhead_stats(h, W, temperature=temperature, softcap=softcap)
    z = h.double() @ W.double().T
    if softcap > 0:
        z = softcap * torch.tanh(z / softcap)
    u = z / temperature
    p = torch.softmax(u, -1)
    np.testing.assert_allclose(logz, torch.logsumexp(u, -1).numpy(), rtol=1e-13)
    np.testing.assert_allclose(H, (-(p * torch.log(p)).sum(-1)).numpy(), rtol=1e-11, atol=1e-13)
    assert np.array_equal(am, u.argmax(-1).numpy())
    top2 = torch.topk(u, 2, -1).values
    np.testing.assert_allclose(gap, (top2[:, 0] - top2[:, 1]).numpy(), rtol=1e-12, atol=1e-14)


def test_uniform_and_peaked_closed_forms():
    d, V = 64, 50
    # identical vocabulary rows: uniform distribution, H = log V, logZ = u + log V
    row = torch.randn(d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    W = row.repeat(V, 1)
    h = torch.randn(2, d, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    logz, H, am, gap = oracle.lmhead_stats(h, W)
    np.testing.assert_allclose(H, math.log(V), rtol=1e-12)
    z = (h.double() @ row.double())
    np.testing.assert_allclose(logz, (z + math.log(V)).numpy(), rtol=1e-12)
    assert np.all(am == 0) and np.all(gap == 0)  # ties go to the lowest index
    # one row far ahead of the rest: H -> 0, argmax is that row
    W2 = torch.zeros(V, d)
    W2[17, 0] = 1.0
    h2 = torch.zeros(1, d)
    h2[0, 0] = 200.0
    logz2, H2, am2, _ = oracle.lmhead_stats(h2.to(torch.bfloat16), W2.to(torch.bfloat16))
    assert am2[0] == 17 and H2[0] < 1e-80 and abs(logz2[0] - 200.0) < 1e-12


def test_lower_temperature_lowers_entropy():
    h, W = _case(T=5, V=200, d=64, seed=5, scale=3.0)
    Hs = [oracle.lmhead_stats(h, W, temperature=t)[1] for t in (1.2, 0.8, 0.4)]
    assert np.all(Hs[0] > Hs[1]) and np.all(Hs[1] > Hs[2])


def _eb_brute(H, masked, bound):
    """Largest k such that the k lowest-entropy masked positions (ties by
    position) have sum minus max <= bound; at least one when any is masked."""
    idx = [t for t in range(len(H)) if masked is None or masked[t]]
    idx.sort(key=lambda t: (H[t], t))
    best = 0
    for k in range(1, len(idx) + 1):
        sel = [H[t] for t in idx[:k]]
        if sum(sel) - max(sel) <= bound:
            best = k
    out = np.zeros(len(H), np.uint8)
    for t in idx[:best]:
        out[t] = 1
    return out


@pytest.mark.parametrize("seed", range(6))
def test_eb_accept_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    T = 40
    H = rng.exponential(0.05, T) * (rng.random(T) < 0.7) + rng.random(T) * (rng.random(T) < 0.3)
    H[rng.integers(0, T, 4)] = H[3]  # ties
    masked = (rng.random(T) < 0.8).astype(np.uint8)
    for bound in (0.0, 0.1, 0.5, 3.0, 1e9):
        got = oracle.eb_accept(H, masked, bound)
        assert np.array_equal(got, _eb_brute(H, masked, bound)), bound
        assert not np.any(got[masked == 0])
        if masked.any():
            assert got.sum() >= 1
    assert np.array_equal(oracle.eb_accept(H, masked, 1e9), masked)
    assert np.array_equal(oracle.eb_accept(H, None, 1e9), np.ones(T, np.uint8))
