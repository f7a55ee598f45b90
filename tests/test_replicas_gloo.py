"""The N>1 host path (replicas, one process per rank) on CPU with gloo,
world size 2: rank environment, barrier, max-over-ranks timing, whole-job
throughput, distinct per-rank inputs, and a missing rank turning into an
error on the others instead of a hang."""
from __future__ import annotations

import os
import socket
import time

import pytest
import torch
import torch.multiprocessing as mp

from block_diffusion_moe_router_b200 import replicas as rep


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})


def _worker_timing(rank, world, port, q):
    _env(rank, world, port)
    r, w = rep.init("gloo", timeout_s=30)
    assert (r, w) == (rank, world)
    # every rank takes the same collective steps: barrier, max, barrier
    rep.barrier()
    ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    mx = rep.max_over_ranks(ms)
    rate = rep.job_rate(256, w, 100, mx)
    from block_diffusion_moe_router_b200 import inputs
    x = inputs._randn((4, 8), 1.0, rep.replica_seed(rank, 0), "cpu", torch.bfloat16)
    rep.barrier()
    q.put((rank, mx, rate, x.float().sum().item()))
    rep.shutdown()


def _worker_missing(rank, world, port, q):
    _env(rank, world, port)
    rep.init("gloo", timeout_s=3)
    if rank == 1:
        q.put((rank, "left"))
        return  # leaves between steps, without joining the next barrier
    t0 = time.time()
    try:
        rep.barrier()
        q.put((rank, "no error"))
    except Exception as e:  # the short process-group timeout ends the wait
        q.put((rank, f"error after {time.time() - t0:.1f}s: {type(e).__name__}"))


def _run(fn, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return sorted(res, key=lambda r: r[0]), [p.exitcode for p in procs]


def test_dist_env_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert rep.dist_env() == (0, 1, 0)
    monkeypatch.setenv("RANK", "3")
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(ValueError):
        rep.dist_env()


def test_single_rank_is_local():
    assert rep.max_over_ranks(7.5) == 7.5
    assert rep.job_rate(256, 1, 10, 1.0) == pytest.approx(256 * 10 / 1e-3)
    with pytest.raises(ValueError):
        rep.job_rate(256, 1, 10, 0.0)


def test_two_ranks_max_and_rate():
    res, codes = _run(_worker_timing, 2)
    assert codes == [0, 0]
    (_, mx0, rate0, s0), (_, mx1, rate1, s1) = res
    assert mx0 == mx1 == 15.0  # the slowest rank's time, on every rank
    assert rate0 == rate1 == pytest.approx(2 * 256 * 100 / 15e-3)
    assert s0 != s1  # replicas draw distinct canvases


def test_missing_rank_raises_not_hangs():
    res, _ = _run(_worker_missing, 2)
    assert res[1][1] == "left"
    assert res[0][1].startswith("error after"), res[0][1]
