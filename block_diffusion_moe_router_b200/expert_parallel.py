"""Expert parallelism of the MoE layer over the ranks of one node.

The pages run the whole model on one device; spreading each layer's 128
experts over N GPUs (rank r owning experts [r*E/N, (r+1)*E/N), every rank
routing its own tokens) is this library's extension.  One layer call is:

  1. route      the rank's tokens                       (router kernel)
  2. dispatch   assignments sorted by owner, x rows packed (plan + gather kernels)
  3. exchange   counts, rows and expert ids, all-to-all  (NCCL / gloo)
  4. experts    the owner's grouped GEMMs on the rows it received
  5. exchange   the y rows back, reverse all-to-all
  6. combine    out_t = residual_t + sum_j w_tj y_(t,j), j in order

Every step of the layer's arithmetic runs in the library's kernels (through
`LibraryOps`); this module moves buffers between them and issues the
collectives.  The collectives use plain torch.distributed all-to-all into
local buffers: no kernel reads another GPU's memory.  Every rank takes the
same collective steps in the same order (four all-to-alls per layer call).

The phases are separate methods (`begin`, `experts`, `finish`) so that a
driver holding all ranks in one process can do the exchanges itself; the
`forward` method chains them with a `TorchExchange` for one process per GPU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch

from . import _abi


def owned_experts(E: int, world: int, rank: int) -> range:
    """Experts of rank `rank`: a contiguous block of E / world."""
    if world < 1 or E % world != 0 or not 0 <= rank < world:
        raise ValueError(f"cannot split {E} experts over {world} ranks (rank {rank})")
    per = E // world
    return range(rank * per, (rank + 1) * per)


def local_slice(t: Optional[torch.Tensor], E: int, world: int, rank: int):
    """The owner's part of a per-expert tensor ([E, ...] row-major, so a
    contiguous view of its first dimension), or None."""
    if t is None:
        return None
    r = owned_experts(E, world, rank)
    return t[r.start:r.stop]


class LibraryOps:
    """The layer's steps on the GPU, through the C ABI: a routing plan (E
    experts, top-k) and an owner plan (the rank's E / world experts, k = 1).
    `chunk_tokens` is the owner plan's MOE_OPT_CHUNK_TOKENS (0: by the size
    of each call); give moe_forward's plan the same explicit value where the
    two must agree byte for byte."""

    def __init__(self, E: int, k: int, d: int, f: int, wdtype: int, world: int,
                 chunk_tokens: int = 0):
        self.E, self.k, self.d, self.f = E, k, d, f
        self.route_plan = _abi.moe_plan_create(E, k, d, f, wdtype)
        self.owner_plan = _abi.moe_plan_create(E // world, 1, d, f, wdtype)
        _abi.moe_plan_set_option(self.owner_plan, _abi.MOE_OPT_CHUNK_TOKENS, chunk_tokens)

    def route(self, x, router_w, router_gamma, router_bias, stream=None):
        T = x.shape[0]
        idx = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        _abi.moe_route(self.route_plan, T, x, router_w, router_gamma, router_bias, idx, w, None,
                       stream)
        return idx, w

    def dispatch(self, x, idx, n_ranks, expert_gamma, stream=None):
        T = x.shape[0]
        A = T * self.k
        send_rows = torch.empty((A, self.d), dtype=torch.bfloat16, device=x.device)
        send_expert = torch.empty(A, dtype=torch.int32, device=x.device)
        pos = torch.empty(A, dtype=torch.int32, device=x.device)
        counts = torch.empty(n_ranks, dtype=torch.int32, device=x.device)
        _abi.moe_ep_dispatch(self.route_plan, T, x, idx, n_ranks, expert_gamma, send_rows,
                             send_expert, pos, counts, stream)
        return send_rows, send_expert, pos, [int(c) for c in counts.cpu()]

    def expert_rows(self, rows, ids, weights, stream=None):
        R = rows.shape[0]
        y = torch.empty((R, self.d), dtype=torch.bfloat16, device=rows.device)
        _abi.moe_expert_rows(self.owner_plan, R, rows, ids, None, weights["w_gate_up"],
                             weights["w_down"], weights.get("scales_gate_up"),
                             weights.get("scales_down"), y, stream)
        return y

    def combine(self, y_rows, pos, w, residual, out, stream=None):
        _abi.moe_combine_rows(self.route_plan, out.shape[0], y_rows, pos, w, residual, out, stream)
        return out

    def status(self, stream=None) -> int:
        a = _abi.moe_plan_sync_status(self.route_plan, stream)
        b = _abi.moe_plan_sync_status(self.owner_plan, stream)
        return a if a != _abi.MOE_OK else b

    def close(self):
        _abi.moe_plan_destroy(self.route_plan)
        _abi.moe_plan_destroy(self.owner_plan)
        self.route_plan = self.owner_plan = None


class TorchExchange:
    """All-to-all of variable-size row blocks over a torch.distributed group
    (NCCL on GPUs, gloo on CPU).  `counts` exchanges the block sizes."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def counts(self, send_counts: List[int], device) -> List[int]:
        s = torch.tensor(send_counts, dtype=torch.int64, device=device)
        r = torch.empty_like(s)
        self.dist.all_to_all_single(r, s, group=self.group)
        return [int(v) for v in r.cpu()]

    def rows(self, send: torch.Tensor, send_counts: List[int], recv_counts: List[int]):
        recv = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype,
                           device=send.device)
        self.dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=recv_counts,
                                    input_split_sizes=send_counts, group=self.group)
        return recv


class LocalExchange:
    """One rank: every block stays where it is."""

    def counts(self, send_counts, device):
        return list(send_counts)

    def rows(self, send, send_counts, recv_counts):
        return send


@dataclass
class Dispatched:
    """What a rank keeps between dispatch and combine."""
    T: int
    w: torch.Tensor          # [T, k] routing weights
    pos: torch.Tensor        # [T*k] send row of each assignment
    send_rows: torch.Tensor  # [T*k, d] rows for the owners, owner-major
    send_expert: torch.Tensor
    send_counts: List[int]


class ExpertParallelLayer:
    """One rank's share of an expert-parallel MoE layer.  `weights` are this
    rank's slices of w_gate_up / w_down (and scales), see `local_slice`."""

    def __init__(self, E: int, k: int, d: int, f: int, wdtype: int = _abi.MOE_W_BF16,
                 rank: int = 0, world: int = 1, exchange=None, ops=None, chunk_tokens: int = 0):
        owned_experts(E, world, rank)  # validates the split
        self.E, self.k, self.d, self.f = E, k, d, f
        self.rank, self.world = rank, world
        self.ops = ops if ops is not None else LibraryOps(E, k, d, f, wdtype, world,
                                                          chunk_tokens)
        if exchange is None:
            exchange = LocalExchange() if world == 1 else TorchExchange()
        self.exchange = exchange

    def begin(self, x, router_w, router_gamma, router_bias=None, expert_gamma=None,
              stream=None) -> Dispatched:
        idx, w = self.ops.route(x, router_w, router_gamma, router_bias, stream)
        send_rows, send_expert, pos, counts = self.ops.dispatch(x, idx, self.world, expert_gamma,
                                                                stream)
        return Dispatched(x.shape[0], w, pos, send_rows, send_expert, counts)

    def experts(self, rows, ids, weights, stream=None):
        return self.ops.expert_rows(rows, ids, weights, stream)

    def finish(self, st: Dispatched, y_back, residual=None, out=None, stream=None):
        if out is None:
            out = torch.empty((st.T, self.d), dtype=torch.bfloat16, device=y_back.device)
        return self.ops.combine(y_back, st.pos, st.w, residual, out, stream)

    def forward(self, x, router_w, router_gamma, weights, router_bias=None, expert_gamma=None,
                residual=None, out=None, stream=None):
        st = self.begin(x, router_w, router_gamma, router_bias, expert_gamma, stream)
        ex = self.exchange
        recv_counts = ex.counts(st.send_counts, x.device)
        rows = ex.rows(st.send_rows, st.send_counts, recv_counts)
        ids = ex.rows(st.send_expert, st.send_counts, recv_counts)
        y = self.experts(rows, ids, weights, stream)
        y_back = ex.rows(y, recv_counts, st.send_counts)
        return self.finish(st, y_back, residual, out, stream)

    def close(self):
        if hasattr(self.ops, "close"):
            self.ops.close()
