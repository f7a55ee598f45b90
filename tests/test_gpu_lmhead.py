"""GPU parity of the lm_head step (logits folded on chip into logZ, entropy
and argmax; entropy-bounded acceptance) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from block_diffusion_moe_router_b200 import inputs
import block_diffusion_moe_router_b200 as moe

pytestmark = pytest.mark.gpu

# fp32 tensor-core accumulation of a d-term dot product and fp32 exp/log:
# logZ and H are good to ~1e-5 relative of the logit scale; 1e-3 absolute
# (plus 1e-4 relative) leaves an order of margin.  The argmax is exact except
# where the oracle's two largest scaled logits are closer than GAP.
TOL_ABS, TOL_REL, GAP = 1e-3, 1e-4, 1e-3


def run(T, V, d, seed, temperature, softcap, bound, masked_frac=0.8, rows=None):
    h, W, _ = inputs.make_lmhead(T, V, d, seed, device="cuda")
    g = torch.Generator().manual_seed(seed)
    masked = (torch.rand(T, generator=g) < masked_frac).to(torch.uint8)
    lh = moe.LmHead(V, d)
    try:
        tok, ent, logz, acc = lh.step(h, W, temperature=temperature, softcap=softcap,
                                      masked=masked.cuda(), entropy_bound=bound)
        assert lh.sync_status() == moe.MOE_OK
    finally:
        lh.close()
    if isinstance(rows, int):  # that many rows spread over the GPU's entropy order
        order = np.argsort(ent.cpu().numpy(), kind="stable")
        rows = np.unique(order[np.linspace(0, T - 1, rows).round().astype(int)])
    rows = np.arange(T) if rows is None else np.asarray(rows)
    olz, oH, oam, ogap = oracle.lmhead_stats(h.cpu(), W.cpu(), rows=rows,
                                             temperature=temperature, softcap=softcap)
    tok, ent, logz, acc = (t.cpu().numpy() for t in (tok, ent, logz, acc))
    np.testing.assert_allclose(logz[rows], olz, rtol=TOL_REL, atol=TOL_ABS)
    np.testing.assert_allclose(ent[rows], oH, rtol=TOL_REL, atol=TOL_ABS)
    clear = ogap >= GAP
    assert np.array_equal(tok[rows][clear], oam[clear])
    # acceptance: the same decision on the same (GPU) entropies, in fp64
    ref_acc = oracle.eb_accept(ent.astype(np.float64), masked.numpy(), bound)
    assert np.array_equal(acc, ref_acc)
    return ent, acc, masked.numpy()


@pytest.mark.parametrize("T,V,d,temperature,softcap", [
    (37, 1000, 256, 0.8, 0.0),     # ragged last vocabulary tile, ragged token slice
    (37, 1000, 256, 0.4, 30.0),    # soft cap, low temperature
    (300, 640, 128, 1.0, 0.0),     # two token chunks
    (1, 128, 64, 0.6, 0.0),        # one token, one tile
])
def test_lmhead_small(T, V, d, temperature, softcap):
    ent, acc, masked = run(T, V, d, seed=T + V, temperature=temperature, softcap=softcap,
                           bound=0.1)
    if masked.any():
        assert acc.sum() >= 1


def test_lmhead_canvas_full_vocab_sampled_rows():
    """The canvas shape: T=256 tokens over a 262144-row vocabulary, d=2816;
    statistics checked on 16 tokens spread evenly over the entropy order, from
    the most peaked to the flattest (the oracle does 0.74 G multiply-adds per
    token), acceptance on all of them."""
    T, V, d = 256, inputs.LMHEAD_V, inputs.LMHEAD_D
    ent, acc, masked = run(T, V, d, seed=5, temperature=0.8, softcap=0.0, bound=0.1, rows=16)
    assert ent.min() < 0.1 and ent.max() > 5.0  # the inputs span peaked to flat


def test_lmhead_bound_extremes_and_determinism():
    T, V, d = 64, 512, 128
    h, W, _ = inputs.make_lmhead(T, V, d, 9, device="cuda")
    lh = moe.LmHead(V, d)
    try:
        a1 = lh.step(h, W, temperature=0.7, entropy_bound=0.0)
        a2 = lh.step(h, W, temperature=0.7, entropy_bound=0.0)
        big = lh.step(h, W, temperature=0.7, entropy_bound=1e30)
        assert lh.sync_status() == moe.MOE_OK
    finally:
        lh.close()
    for x, y in zip(a1, a2):
        assert torch.equal(x, y)
    assert int(a1[3].sum()) >= 1          # bound 0: the lowest entropy (and exact ties to 0)
    assert int(big[3].sum()) == T         # no mask, unbounded: everything accepted


def test_lmhead_invalid_arguments():
    lh = moe.LmHead(256, 128)
    h = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(256, 128, dtype=torch.bfloat16, device="cuda")
    out = [torch.empty(4, dtype=dt, device="cuda") for dt in (torch.int32, torch.float32,
                                                               torch.float32, torch.uint8)]
    try:
        for temp, cap, bound in [(0.0, 0.0, 0.1), (-1.0, 0.0, 0.1), (1.0, -1.0, 0.1),
                                 (1.0, 0.0, -0.5), (float("nan"), 0.0, 0.1)]:
            st = moe.moe_lmhead_forward(lh.handle, 4, h, W, temp, cap, None, bound, *out,
                                        check=False)
            assert st == moe.MOE_ERR_INVALID_ARG
        st = moe.moe_lmhead_forward(lh.handle, 5000, h, W, 1.0, 0.0, None, 0.1, *out, check=False)
        assert st == moe.MOE_ERR_INVALID_ARG
        assert moe.moe_lmhead_forward(lh.handle, 0, h, W, 1.0, 0.0, None, 0.1, *out) == moe.MOE_OK
    finally:
        lh.close()
