"""Expert parallelism for the int4 MoE layer: the routed experts sharded over the ranks of a
process group, one GPU per rank.

The layer is the one include/moe.h defines (router softmax over E experts, top-k plus a sigmoid-gated
shared expert, SwiGLU experts with int4 group-64 weights).  With W ranks, rank r holds routed experts
[r E/W, (r+1) E/W) and a replica of the router and of the shared expert.  One forward call on a rank's
own tokens x[T, H]:

1. route (libmoe ``moe_route`` on a router-only handle): idx[T, k], gates[T, k], shared gate[T];
2. plan: the T*k (token, slot) pairs sorted stably by destination rank = idx // (E/W); counts per rank;
3. exchange the counts, then the pairs' rows (bf16, gathered by libmoe) and their (local expert id,
   gate) with all-to-all;
4. experts (libmoe ``moe_forward_routed`` on this rank's expert handle, one slot per row): every row
   received -> gate x FFN(row) in bf16; and the shared expert on this rank's own tokens (a one-expert
   handle, gated by the shared gate);
5. return the received rows' results to their source ranks (all-to-all, the reverse split);
6. combine (libmoe ``moe_combine_rows``): out[t] = bf16(shared result[t] + sum_j returned[t, j]), fp32 sums.

Steps 3 and 5 are the only exchanges; they use ``torch.distributed.all_to_all_single`` (NCCL on GPUs,
gloo on CPU), whose split sizes live on the host, so a call reads the W receive counts back once.
Index bookkeeping (the sort by rank, the inverse positions) is host logic on small int tensors; every
step that touches activations or weights runs in libmoe.

The compute steps go through a ``shard`` object (route / gather / experts / combine), so the plan
and the exchange can be exercised on CPU ranks with any implementation of those four steps.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import torch


@dataclass
class DispatchPlan:
    """Where each (token, slot) pair of one rank's call goes.

    order:       [P] int64, flat pair index t*k + j, sorted by destination rank (stable: within a rank,
                 pairs keep token-then-slot order); P = T*k
    send_counts: [W] int64, pairs sent to each rank (in ``order``, rank 0's first)
    pair_token:  [P] int64, the token of each pair in ``order``
    local_ids:   [P] int32, the pair's expert id on its destination rank (idx - rank * E/W)
    gates:       [P] fp32, the pair's gate
    pos:         [T, k] int32, position of pair (t, j) in ``order`` (the inverse permutation)
    """
    order: torch.Tensor
    send_counts: torch.Tensor
    pair_token: torch.Tensor
    local_ids: torch.Tensor
    gates: torch.Tensor
    pos: torch.Tensor


def plan_dispatch(idx: torch.Tensor, gates: torch.Tensor, experts_per_rank: int, world: int) -> DispatchPlan:
    """Sort one rank's (token, slot) pairs by the rank that holds their expert."""
    T, k = idx.shape
    flat = idx.reshape(-1).to(torch.int64)
    if flat.numel() and (int(flat.min()) < 0 or int(flat.max()) >= experts_per_rank * world):
        raise ValueError("expert id outside [0, E)")
    dest = torch.div(flat, experts_per_rank, rounding_mode="floor")
    order = torch.argsort(dest, stable=True)
    send_counts = torch.bincount(dest, minlength=world)
    pair_token = torch.div(order, k, rounding_mode="floor")
    local_ids = (flat[order] - dest[order] * experts_per_rank).to(torch.int32)
    pos = torch.empty_like(order)
    pos[order] = torch.arange(order.numel(), device=order.device)
    return DispatchPlan(order=order, send_counts=send_counts, pair_token=pair_token, local_ids=local_ids,
                        gates=gates.reshape(-1)[order].to(torch.float32).contiguous(),
                        pos=pos.view(T, k).to(torch.int32).contiguous())


class Exchange:
    """All-to-all with variable splits over a torch.distributed group (None: no group, one rank)."""

    def __init__(self, group=None, world: int = 1):
        self.group = group
        self.world = world

    def counts(self, send_counts: torch.Tensor) -> torch.Tensor:
        if self.world == 1:
            return send_counts.clone()
        import torch.distributed as dist
        recv = torch.empty_like(send_counts)
        dist.all_to_all_single(recv, send_counts, group=self.group)
        return recv

    def rows(self, send: torch.Tensor, send_splits, recv_splits, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """send[sum(send_splits), ...] -> out[sum(recv_splits), ...]; splits are host int lists."""
        n = int(sum(recv_splits))
        if out is None:
            out = torch.empty((n,) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        if self.world == 1:
            out.copy_(send)
            return out
        import torch.distributed as dist
        dist.all_to_all_single(out, send, output_split_sizes=list(recv_splits),
                               input_split_sizes=list(send_splits), group=self.group)
        return out


_EXPERT_FIELDS = ("q_gate", "q_up", "q_down", "s_gate", "b_gate", "s_up", "b_up", "s_down", "b_down")
_SHARED_FIELDS = ("qs_gate", "qs_up", "qs_down", "ss_gate", "bs_gate", "ss_up", "bs_up", "ss_down", "bs_down")


class LibraryShard:
    """One rank's compute steps on its GPU, all in libmoe: a router-only handle (router, bias and
    shared gate over all E experts), an expert handle holding this rank's E/W routed experts (top-k
    1, no router) and a one-expert handle holding the shared expert."""

    def __init__(self, weights: Dict[str, torch.Tensor], H: int, I: int, E: int, k: int, has_shared: bool,
                 rank: int, world: int, max_tokens: int = 4096, max_rows: Optional[int] = None,
                 device=None, stream=None):
        from . import _lib as M
        if E % world:
            raise ValueError(f"{E} experts do not split evenly over {world} ranks")
        self.H, self.E, self.k, self.has_shared = H, E, k, bool(has_shared)
        self.n_local = E // world
        e0 = rank * self.n_local
        rw = {n: weights.get(n) for n in ("router", "router_bias", "shared_gate")}
        self.router = M.Layer(rw, H, I, E, k, has_shared, max_tokens=max_tokens, decode_max_tokens=0,
                              flags=M.MOE_FLAG_NO_EXPERTS, device=device, stream=stream)
        # this rank's routed experts (top-k 1: one expert per row); the shared expert in a handle of
        # its own (expert 0 of 1), gated per token by the router's shared gate
        ew = {n: weights[n][e0:e0 + self.n_local].contiguous() for n in _EXPERT_FIELDS}
        # every row of every rank could come here (W*T*k); larger exchanges run in slices of max_rows
        self.max_rows = max_rows or min(65536, world * max_tokens * k)
        self.experts = M.Layer(ew, H, I, self.n_local, 1, False, max_tokens=self.max_rows, decode_max_tokens=0,
                               flags=M.MOE_FLAG_NO_ROUTER, device=device, stream=stream)
        del ew
        self.shared = None
        if has_shared:
            sw = {n: weights[ns].unsqueeze(0).contiguous() for n, ns in zip(_EXPERT_FIELDS, _SHARED_FIELDS)}
            self.shared = M.Layer(sw, H, I, 1, 1, False, max_tokens=max_tokens, decode_max_tokens=0,
                                  flags=M.MOE_FLAG_NO_ROUTER, device=device, stream=stream)
            del sw

    def route(self, x):
        r = self.router.route(x)
        return r["idx"], r["gates"], (r["shared_gate"] if self.has_shared else None)

    def gather(self, x, rows):
        """x[rows] through libmoe (a one-term combine is an exact bf16 copy)."""
        return self.router.combine_rows(x, rows.to(torch.int32).view(-1, 1).contiguous())

    def experts_forward(self, rows, ids, gates):
        """gate x FFN_id(row) for every row, bf16 [n, H]; ids index this rank's routed experts."""
        n = rows.shape[0]
        out = torch.empty((n, self.H), dtype=torch.bfloat16, device=rows.device)
        step = max(64, self.max_rows // 64 * 64)   # 16-byte aligned slices of ids and gates
        for s in range(0, n, step):
            e = min(n, s + step)
            self.experts.forward_routed(rows[s:e], ids[s:e].view(-1, 1), gates[s:e].view(-1, 1), out=out[s:e])
        return out

    def shared_forward(self, x, shared_gate):
        """shared_gate x FFN_shared(x) for the rank's own tokens, bf16 [T, H] (None without one)."""
        if self.shared is None:
            return None
        ids = torch.zeros((x.shape[0], 1), dtype=torch.int32, device=x.device)
        return self.shared.forward_routed(x, ids, shared_gate.view(-1, 1).contiguous())

    def combine(self, returned, pos, base):
        return self.router.combine_rows(returned, pos, base=base)

    def close(self):
        for L in (self.router, self.experts, self.shared):
            if L is not None:
                L.close()


class ExpertParallelLayer:
    """One MoE layer with its routed experts sharded over ``exchange.world`` ranks.

    ``shard`` runs the compute steps on this rank (``LibraryShard``: libmoe on the rank's GPU);
    ``exchange`` moves rows between ranks.  Every rank calls ``forward`` on its own tokens, in the same
    order as the other ranks (the exchanges are collective)."""

    def __init__(self, shard, exchange: Exchange):
        self.shard = shard
        self.exchange = exchange
        self.world = exchange.world
        self.n_local = shard.n_local

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        sh, ex = self.shard, self.exchange
        idx, gates, sg = sh.route(x)                                           # 1
        plan = plan_dispatch(idx, gates, self.n_local, self.world)             # 2
        recv_counts = ex.counts(plan.send_counts)                              # 3
        send_splits = plan.send_counts.tolist()
        recv_splits = recv_counts.tolist()
        x_send = sh.gather(x, plan.pair_token)
        meta = torch.stack([plan.local_ids, plan.gates.view(torch.int32)], 1).contiguous()
        x_recv = ex.rows(x_send, send_splits, recv_splits)
        meta_recv = ex.rows(meta, send_splits, recv_splits)
        ids = meta_recv[:, 0].contiguous()
        g = meta_recv[:, 1].contiguous().view(torch.float32)
        y_recv = sh.experts_forward(x_recv, ids, g)                            # 4
        y_shared = sh.shared_forward(x, sg) if sg is not None else None
        returned = ex.rows(y_recv, recv_splits, send_splits)                   # 5
        return sh.combine(returned, plan.pos, y_shared)                        # 6
