"""Expert parallelism on CPU: the orchestration of
block_diffusion_moe_router_b200.expert_parallel (dispatch plan, count and
row all-to-alls over gloo, the owner's rows, the return all-to-all and the
combine) at world sizes 2 and 4, one process per rank.

The layer's steps run in a CPU stand-in for the GPU kernels built on the
oracle (routing, one expert on one row, the weighted sum in j order), so
what is checked here is the part the GPU cannot be used for on this machine:
that every assignment reaches its owner, comes back to the right slot, and
that the result does not depend on the number of ranks (bit-identical to one
rank) and equals the oracle's whole layer.  The same orchestration drives
the library's kernels in the GPU tests.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from block_diffusion_moe_router_b200 import inputs
from block_diffusion_moe_router_b200 import expert_parallel as ep

T, E, K, D, F = 24, 8, 3, 128, 64


class OracleOps:
    """The layer's steps on the CPU, with the contracts of LibraryOps: rows
    travel as float64 copies of the bf16 inputs."""

    def __init__(self, E, k, world, layer):
        self.E, self.k, self.world = E, k, world
        self.per = E // world
        self.layer = layer

    def route(self, x, router_w, router_gamma, router_bias, stream=None):
        idx, w, _, _ = oracle.route(x, router_w, router_gamma, router_bias, self.k)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def dispatch(self, x, idx, n_ranks, expert_gamma, stream=None):
        assert expert_gamma is None
        flat = idx.reshape(-1).numpy()
        owner = flat // self.per
        order = np.argsort(owner, kind="stable")          # send row -> assignment
        pos = np.empty_like(order)
        pos[order] = np.arange(order.size)
        xs = oracle.decode_bf16(x)
        send_rows = torch.from_numpy(xs[order // self.k])
        send_expert = torch.from_numpy((flat[order] % self.per).astype(np.int32))
        counts = np.bincount(owner, minlength=n_ranks).tolist()
        return send_rows, send_expert, torch.from_numpy(pos.astype(np.int32)), counts

    def expert_rows(self, rows, ids, weights, stream=None):
        y = np.empty((rows.shape[0], rows.shape[1]), np.float64)
        for r in range(rows.shape[0]):
            y[r], _ = oracle.expert_ffn(rows[r].numpy(), int(ids[r]), weights["w_gate_up"],
                                        weights["w_down"])
        return torch.from_numpy(y)

    def combine(self, y_rows, pos, w, residual, out, stream=None):
        Tl = w.shape[0]
        y = y_rows.numpy()
        p = pos.numpy().reshape(Tl, self.k)
        o = np.zeros((Tl, y.shape[1])) if residual is None else oracle.decode_bf16(residual)
        for t in range(Tl):
            for j in range(self.k):
                o[t] = o[t] + w[t, j].item() * y[p[t, j]]
        out.copy_(torch.from_numpy(o))
        return out


def _layer():
    lay = inputs.make_small(T=T, d=D, E=E, k=K, f=F, seed=606, bias=True, residual=True)
    return lay


def _run_rank(rank, world, lay, exchange):
    rows = slice(rank * T // world, (rank + 1) * T // world)
    ops = OracleOps(E, K, world, lay)
    layer = ep.ExpertParallelLayer(E, K, D, F, rank=rank, world=world, exchange=exchange, ops=ops)
    weights = {"w_gate_up": ep.local_slice(lay["w_gate_up"], E, world, rank),
               "w_down": ep.local_slice(lay["w_down"], E, world, rank)}
    x = lay["x"][rows].contiguous()
    res = lay["residual"][rows].contiguous()
    out = torch.empty((x.shape[0], D), dtype=torch.float64)
    layer.forward(x, lay["router_w"], lay["router_gamma"], weights,
                  router_bias=lay["router_bias"], residual=res, out=out)
    return out.numpy()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out = _run_rank(rank, world, _layer(), ep.TorchExchange())
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def _spawn(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in procs] == [0] * world
    return np.concatenate([res[r] for r in range(world)])


@pytest.fixture(scope="module")
def single_rank():
    lay = _layer()
    return lay, _run_rank(0, 1, lay, ep.LocalExchange())


def test_one_rank_equals_the_oracle_layer(single_rank):
    lay, got = single_rank
    ref, _, _, _ = oracle.moe_forward(lay["x"], lay["router_w"], lay["router_gamma"],
                                      lay["router_bias"], lay["w_gate_up"], lay["w_down"], K,
                                      residual=lay["residual"])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("world", [2, 4])
def test_ranks_over_gloo_bit_identical_to_one_rank(single_rank, world):
    _, want = single_rank
    got = _spawn(world)
    assert np.array_equal(got, want)


def test_dispatch_plan_is_owner_major_and_stable():
    """Every owner's rows are contiguous, in (token, j) order, and pos maps
    each assignment to its own row."""
    lay = _layer()
    ops = OracleOps(E, K, 4, lay)
    idx, _ = ops.route(lay["x"], lay["router_w"], lay["router_gamma"], lay["router_bias"])
    rows, ids, pos, counts = ops.dispatch(lay["x"], idx, 4, None)
    flat = idx.reshape(-1).numpy()
    assert sum(counts) == T * K
    start = np.concatenate([[0], np.cumsum(counts)])
    for r in range(4):
        seg = [a for a in range(T * K) if start[r] <= pos[a] < start[r + 1]]
        assert all(flat[a] // (E // 4) == r for a in seg)
        assert [int(pos[a]) for a in seg] == list(range(start[r], start[r + 1]))
        for a in seg:
            assert int(ids[pos[a]]) == flat[a] % (E // 4)


def test_owned_experts_and_slices():
    assert list(ep.owned_experts(128, 8, 3)) == list(range(48, 64))
    w = torch.arange(8 * 2).reshape(8, 2)
    assert torch.equal(ep.local_slice(w, 8, 4, 1), w[2:4])
    with pytest.raises(ValueError):
        ep.owned_experts(128, 3, 0)
