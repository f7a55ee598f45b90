"""Expert parallelism on the GPU, through the C ABI (moe_route,
moe_ep_dispatch, moe_expert_rows, moe_combine_rows) and the orchestration in
block_diffusion_moe_router_b200.expert_parallel.  An expert's tokens form the
same chunks on an owner as in moe_forward and the kernels' arithmetic for a
chunk depends on that chunk alone, so the bytes must agree:

  - one rank: bit-identical to moe_forward on the same inputs;
  - four ranks emulated in one process on one GPU (the all-to-alls done by
    concatenating the ranks' buffers, every kernel launched in turn, none
    waiting on another): each rank's tokens bit-identical to moe_forward on
    the whole canvas;
  - the dispatch plan against a stable sort by owner.
"""
import numpy as np
import pytest
import torch

import block_diffusion_moe_router_b200 as moe
from block_diffusion_moe_router_b200 import expert_parallel as ep
from block_diffusion_moe_router_b200 import inputs

pytestmark = pytest.mark.gpu


def _cuda(lay):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}


def _reference(lay, E, k, d, f, wd, residual, chunk_tokens=0):
    layer = moe.MoeLayer(E, k, d, f, wd)
    try:
        moe.moe_plan_set_option(layer.plan, moe.MOE_OPT_CHUNK_TOKENS, chunk_tokens)
        out = layer.forward(lay["x"], lay["router_w"], lay["router_gamma"], lay["w_gate_up"],
                            lay["w_down"], router_bias=lay.get("router_bias"),
                            scales_gate_up=lay.get("scales_gate_up"),
                            scales_down=lay.get("scales_down"), residual=residual,
                            expert_gamma=lay.get("expert_gamma"))
        assert layer.sync_status() == moe.MOE_OK
        return out.clone()
    finally:
        layer.close()


def _weights(lay, E, world, rank):
    return {key: ep.local_slice(lay.get(key), E, world, rank)
            for key in ("w_gate_up", "w_down", "scales_gate_up", "scales_down")}


def _emulated(lay, E, k, d, f, wd, world, residual, chunk_tokens=0):
    """All ranks in this process: phases in turn, exchanges by concatenation."""
    T = lay["x"].shape[0]
    sl = [slice(r * T // world, (r + 1) * T // world) for r in range(world)]
    layers = [ep.ExpertParallelLayer(E, k, d, f, wd, rank=r, world=world,
                                     exchange=ep.LocalExchange(), chunk_tokens=chunk_tokens)
              for r in range(world)]
    try:
        st = [layers[r].begin(lay["x"][sl[r]].contiguous(), lay["router_w"], lay["router_gamma"],
                              lay.get("router_bias"), lay.get("expert_gamma"))
              for r in range(world)]
        start = [np.concatenate([[0], np.cumsum(s.send_counts)]) for s in st]
        ys = []
        for o in range(world):  # owner o receives block o of every rank, in rank order
            rows = torch.cat([st[r].send_rows[start[r][o]:start[r][o + 1]] for r in range(world)])
            ids = torch.cat([st[r].send_expert[start[r][o]:start[r][o + 1]]
                             for r in range(world)])
            ys.append(layers[o].experts(rows, ids, _weights(lay, E, world, o)))
        outs = []
        for r in range(world):  # rank r gets its block back from every owner
            back = []
            for o in range(world):
                before = sum(st[q].send_counts[o] for q in range(r))
                back.append(ys[o][before:before + st[r].send_counts[o]])
            res = residual[sl[r]].contiguous() if residual is not None else None
            outs.append(layers[r].finish(st[r], torch.cat(back), residual=res))
        for L in layers:
            assert L.ops.status() == moe.MOE_OK
        return torch.cat(outs)
    finally:
        for L in layers:
            L.close()


@pytest.mark.parametrize("wd", [inputs.WDTYPE_BF16, inputs.WDTYPE_INT4])
def test_one_rank_bit_identical_to_moe_forward(wd):
    T, E, k, d, f = 96, 16, 4, 256, 128
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=700 + wd, wdtype=wd, bias=True,
                                  residual=True, expert_norm=True))
    want = _reference(lay, E, k, d, f, wd, lay["residual"])
    layer = ep.ExpertParallelLayer(E, k, d, f, wd)
    try:
        got = layer.forward(lay["x"], lay["router_w"], lay["router_gamma"], _weights(lay, E, 1, 0),
                            router_bias=lay["router_bias"], expert_gamma=lay["expert_gamma"],
                            residual=lay["residual"])
        assert layer.ops.status() == moe.MOE_OK
    finally:
        layer.close()
    assert torch.equal(got, want)


@pytest.mark.parametrize("chunk_tokens", [128, 256])
def test_four_emulated_ranks_on_the_canvas(chunk_tokens):
    """The canvas layer (T=256, d=2816, 128 experts, top-8, f=704) over four
    emulated ranks of 64 tokens and 32 experts each, with a residual and a
    router bias that sends every token to expert 5 (two 128-token chunks, or
    one 256-token chunk, next to small ones).  The owners' plans and the
    reference plan take the same explicit chunk size: by default it follows
    each call's size, and an owner's call (all rows it receives) is not the
    size of the whole layer's."""
    w = inputs.WORKLOADS["canvas"]
    lay = inputs.make_layer(w, device="cuda")
    lay["router_bias"] = torch.zeros(w.E, device="cuda")
    lay["router_bias"][5] = 50.0
    res = inputs._randn((w.T, w.d), 1.0, 78, "cuda", torch.bfloat16)
    want = _reference(lay, w.E, w.k, w.d, w.f, inputs.WDTYPE_BF16, res, chunk_tokens)
    got = _emulated(lay, w.E, w.k, w.d, w.f, inputs.WDTYPE_BF16, 4, res, chunk_tokens)
    assert torch.equal(got, want)


@pytest.mark.parametrize("world", [2, 8])
def test_emulated_ranks_small(world):
    T, E, k, d, f = 77, 16, 4, 384, 192
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=80 + world, bias=True,
                                  expert_norm=True))
    want = _reference(lay, E, k, d, f, inputs.WDTYPE_BF16, None)
    got = _emulated(lay, E, k, d, f, inputs.WDTYPE_BF16, world, None)
    assert torch.equal(got, want)


def test_dispatch_plan_matches_a_stable_sort_by_owner():
    T, E, k, d, f = 130, 32, 5, 256, 64
    lay = _cuda(inputs.make_small(T=T, d=d, E=E, k=k, f=f, seed=90, bias=True))
    n = 4
    ops = ep.LibraryOps(E, k, d, f, inputs.WDTYPE_BF16, n)
    try:
        idx, _ = ops.route(lay["x"], lay["router_w"], lay["router_gamma"], lay["router_bias"])
        rows, ids, pos, counts = ops.dispatch(lay["x"], idx, n, None)
        assert ops.status() == moe.MOE_OK
    finally:
        ops.close()
    flat = idx.reshape(-1).cpu().numpy()
    per = E // n
    order = np.argsort(flat // per, kind="stable")
    want_pos = np.empty_like(order)
    want_pos[order] = np.arange(order.size)
    assert counts == np.bincount(flat // per, minlength=n).tolist()
    assert np.array_equal(pos.cpu().numpy(), want_pos)
    assert np.array_equal(ids.cpu().numpy(), flat[order] % per)
    assert torch.equal(rows, lay["x"][torch.as_tensor(order // k, device="cuda")])


def test_combine_rows_clamps_and_reports_a_bad_position():
    T, E, k, d, f = 8, 16, 2, 256, 64
    plan = moe.moe_plan_create(E, k, d, f)
    try:
        y = torch.ones((T * k, d), dtype=torch.bfloat16, device="cuda")
        w = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
        pos = torch.arange(T * k, dtype=torch.int32, device="cuda")
        pos[3] = T * k + 5  # outside the rows
        out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        moe.moe_combine_rows(plan, T, y, pos, w, None, out)
        assert moe.moe_plan_sync_status(plan) == moe.MOE_ERR_DEVICE_CHECK
        assert torch.equal(out, torch.ones_like(out))  # every row still 0.5 + 0.5
    finally:
        moe.moe_plan_destroy(plan)
