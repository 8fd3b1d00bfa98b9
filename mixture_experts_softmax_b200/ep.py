"""Expert parallelism: the MoE layer with its experts spread over W ranks.

The pages' own model spreads the experts over the devices of the `model` mesh axis
("Grok-1 Admin & Architecture Guide", section 6 "Sharding & Parallelism Deep Dive":
the MoE matmuls run under shard_map and a psum adds the partial results).  Here rank r
of W holds the E/W consecutive experts [r*E/W, (r+1)*E/W) and its own tokens, and one
layer is

    moe_ep_dispatch  (device)   route the rank's tokens; rows grouped by expert
    exchange counts  (all-to-all of E/W ints per rank pair)
    exchange rows    (all-to-all of bf16 rows, variable sizes)
    moe_ep_experts   (device)   the rank's experts on the rows it received
    exchange y rows  (the reverse all-to-all, fp32)
    moe_ep_combine   (device)   gate-weighted sum back in token order

Each device step is a call of the C ABI (include/moe.h); this module holds the
exchange plan and the exchanges: ``torch.distributed.all_to_all_single`` over a
process group (NCCL on GPUs, gloo on the host), or, for one process that drives the
state of several ranks (tests on one GPU), ``local_all_to_all``.  ``ep_forward``
composes the steps and is the same code for both.
"""
from __future__ import annotations

from typing import Callable, List, Sequence, Tuple

import torch

from . import (MOE_LAYOUT_PACKED, MoELayer, check, moe_ep_combine, moe_ep_dispatch, moe_ep_experts,
               moe_set_weight_layout, pack_layer)


def expert_range(E: int, world: int, rank: int) -> Tuple[int, int]:
    """The experts [first, last) that `rank` of `world` holds."""
    if world < 1 or E % world:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    El = E // world
    return rank * El, (rank + 1) * El


def plan_exchange(send_counts: Sequence[int], recv_counts: Sequence[Sequence[int]], world: int):
    """Row counts of the two exchanges of one rank.

    send_counts: this rank's routed rows per expert [E]; recv_counts: [world][E/world], the
    rows each source rank sends for this rank's experts.  Returns (send_splits, recv_splits):
    rows to each destination rank (its experts' counts, in expert order, which is the order
    of send_rows) and rows from each source rank.  The reverse exchange swaps the two."""
    E = len(send_counts)
    _, El = expert_range(E, world, 0)
    send_splits = [int(sum(send_counts[j * El:(j + 1) * El])) for j in range(world)]
    recv_splits = [int(sum(recv_counts[s])) for s in range(world)]
    return send_splits, recv_splits


def dist_all_to_all(group=None) -> Callable:
    """all_to_all(send, send_splits, recv_splits) over a torch.distributed process group."""
    import torch.distributed as dist

    def a2a(send: torch.Tensor, send_splits: List[int], recv_splits: List[int]) -> torch.Tensor:
        out = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        dist.all_to_all_single(out, send[:sum(send_splits)].contiguous(), recv_splits, send_splits, group=group)
        return out
    return a2a


def local_all_to_all(sends: List[torch.Tensor], send_splits: List[List[int]]) -> List[torch.Tensor]:
    """The all-to-all of W ranks whose buffers one process holds: rank r receives, from every
    source s in rank order, the send_splits[s][r] rows that follow s's rows for ranks < r."""
    W = len(sends)
    outs = []
    for r in range(W):
        parts = []
        for s in range(W):
            a = sum(send_splits[s][:r])
            parts.append(sends[s][a:a + send_splits[s][r]])
        outs.append(torch.cat(parts, dim=0))
    return outs


def ep_forward(dispatch: Callable, experts: Callable, combine: Callable, world: int, E: int, group=None):
    """One expert-parallel layer on this rank over a process group.

    dispatch() -> (send_rows [>= n, d], send_counts [E] int32); experts(recv_counts [world,
    E/world] host int32, recv_rows [R, d]) -> y [R, d]; combine(y_back [n, d]).  The counts
    exchange is an equal-split all-to-all of E/world ints per rank pair; its result is read on
    the host, since the row exchanges need their sizes."""
    import torch.distributed as dist
    _, El = expert_range(E, world, 0)
    send_rows, send_counts = dispatch()
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts.contiguous(), group=group)
    sc = send_counts.cpu().tolist()
    rc = recv_counts.cpu().view(world, El)
    send_splits, recv_splits = plan_exchange(sc, rc.tolist(), world)
    a2a = dist_all_to_all(group)
    recv_rows = a2a(send_rows, send_splits, recv_splits)
    y = experts(rc, recv_rows)
    y_back = a2a(y, recv_splits, send_splits)
    return combine(y_back)


class EPRank:
    """One rank's part of the expert-parallel layer: a handle plus the rank's experts.

    local_layer: dict with router_w (the full [d, E] router) and the rank's experts' wl, sl,
    wv, sv, w1, s1 ([E/world, ...], drawn [E, in, out] orientation); with packed=True they
    are repacked once here to the TMEM path's layout."""

    def __init__(self, d: int, ffn: int, world: int, rank: int, local_layer: dict, E: int = 8,
                 packed: bool = True):
        self.d, self.ffn, self.E, self.world, self.rank = d, ffn, E, world, rank
        self.first, self.last = expert_range(E, world, rank)
        self.E_local = self.last - self.first
        self.layer = MoELayer(d, ffn, E, 2)
        if packed:
            check(moe_set_weight_layout(self.layer.h, MOE_LAYOUT_PACKED), "moe_set_weight_layout")
            local_layer = pack_layer(self.layer.h, local_layer)
        self.w = local_layer
        self.T = 0

    def close(self):
        self.layer.close()

    def dispatch(self, x: torch.Tensor, stream=None):
        T = x.shape[0]
        self.T = T
        send_rows = torch.empty((2 * T, self.d), dtype=torch.bfloat16, device=x.device)
        send_counts = torch.empty(self.E, dtype=torch.int32, device=x.device)
        check(moe_ep_dispatch(self.layer.h, T, x, self.w["router_w"], send_rows, send_counts, stream),
              "moe_ep_dispatch")
        return send_rows, send_counts

    def experts(self, recv_counts, recv_rows: torch.Tensor, stream=None) -> torch.Tensor:
        rc = torch.as_tensor(recv_counts, dtype=torch.int32).cpu().view(-1, self.E_local)
        R = int(rc.sum())
        y = torch.empty((R, self.d), dtype=torch.float32, device=recv_rows.device)
        w = self.w
        check(moe_ep_experts(self.layer.h, rc.shape[0], self.E_local, rc, recv_rows, w["wl"], w["sl"], w["wv"],
                             w["sv"], w["w1"], w["s1"], y, stream), "moe_ep_experts")
        return y

    def combine(self, y_back: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
        check(moe_ep_combine(self.layer.h, self.T, y_back, out, stream), "moe_ep_combine")
        return out

    def forward(self, x: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
        """The layer on this rank's tokens, with the other ranks of `group` (torch.distributed)."""
        return ep_forward(lambda: self.dispatch(x), lambda rc, rows: self.experts(rc, rows),
                          lambda yb: self.combine(yb, out), self.world, self.E, group)


def forward_local(ranks: List[EPRank], xs: List[torch.Tensor], outs: List[torch.Tensor]):
    """All ranks' layers driven from one process (the ranks' handles may share one GPU): the
    same steps as EPRank.forward, with local_all_to_all as the exchange.  No kernel of one
    rank waits for another's: the steps run rank after rank."""
    W = len(ranks)
    E = ranks[0].E
    El = E // W
    sent = [rk.dispatch(x) for rk, x in zip(ranks, xs)]
    counts = [sc.cpu() for _, sc in sent]
    recv_counts = [torch.stack([counts[s][r * El:(r + 1) * El] for s in range(W)]) for r in range(W)]
    plans = [plan_exchange(counts[r].tolist(), recv_counts[r].tolist(), W) for r in range(W)]
    recv_rows = local_all_to_all([rows for rows, _ in sent], [p[0] for p in plans])
    ys = [rk.experts(recv_counts[r], recv_rows[r]) for r, rk in enumerate(ranks)]
    y_back = local_all_to_all(ys, [p[1] for p in plans])
    return [rk.combine(yb, out) for rk, yb, out in zip(ranks, y_back, outs)]


def slice_experts(layer: dict, first: int, last: int) -> dict:
    """The rank's share of a full layer: the router whole, the experts [first, last)."""
    out = {"router_w": layer["router_w"]}
    for k in ("wl", "sl", "wv", "sv", "w1", "s1"):
        out[k] = layer[k][first:last].contiguous()
    return out
