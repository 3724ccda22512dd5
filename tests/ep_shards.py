"""Test implementations of the four compute steps of an expert-parallel layer (route, gather,
experts, combine), for running bit_grouped_expert_router_b200.ep on CPU ranks:

OracleShard  the layer's arithmetic from the CPU oracle (fp64, each returned row rounded to bf16 as
             the library's rows are), so a multi-rank result can be compared with the oracle's
             single-process forward;
LabelShard   exact arithmetic on labelled rows (float64 row = token label, expert output = label x
             (global expert id + 1) x gate), so every row's trip to its expert and back is checked
             bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch


class OracleShard:
    def __init__(self, ol, rank: int, world: int):
        self.ol = ol
        self.E, self.k, self.H = ol.E, ol.k, ol.H
        self.n_local = ol.E // world
        self.e0 = rank * self.n_local
        self.has_shared = ol.has_shared

    def route(self, x):
        idx, g, sg, _ = self.ol.route(x)
        return (torch.from_numpy(idx).to(torch.int32), torch.from_numpy(g).to(torch.float32),
                torch.from_numpy(sg).to(torch.float32) if self.has_shared else None)

    def gather(self, x, rows):
        return x[rows.to(torch.int64)]

    def _ffn_rows(self, experts, rows, gates):
        xs = rows.to(torch.float64).numpy()
        out = np.zeros((rows.shape[0], self.H), np.float64)
        for i in range(rows.shape[0]):
            out[i] = float(gates[i]) * self.ol.expert_ffn(int(experts[i]), xs[i])
        return torch.from_numpy(out).to(torch.bfloat16)

    def experts_forward(self, rows, ids, gates):
        return self._ffn_rows(ids.to(torch.int64) + self.e0, rows, gates)

    def shared_forward(self, x, sg):
        return self._ffn_rows(torch.full((x.shape[0],), self.E), x, sg)

    def combine(self, returned, pos, base):
        acc = base.to(torch.float32) if base is not None else torch.zeros((pos.shape[0], self.H))
        for j in range(pos.shape[1]):
            acc = acc + returned[pos[:, j].to(torch.int64)].to(torch.float32)
        return acc.to(torch.bfloat16)


class LabelShard:
    E, k = 16, 3

    def __init__(self, rank: int, world: int):
        self.rank = rank
        self.n_local = self.E // world
        self.e0 = rank * self.n_local

    @staticmethod
    def routing(rank: int, T: int, E: int, k: int):
        t = torch.arange(T).view(-1, 1)
        j = torch.arange(k).view(1, -1)
        idx = ((t * 7 + j * 5 + rank * 3) % E).to(torch.int32)
        gates = (0.5 ** j.to(torch.float32)).expand(T, k).contiguous()
        sg = torch.full((T,), 0.25)
        return idx, gates, sg

    @staticmethod
    def tokens(rank: int, T: int):
        x = torch.zeros((T, 4), dtype=torch.float64)
        x[:, 0] = rank * 1000 + torch.arange(T, dtype=torch.float64)
        x[:, 1] = 1.0
        return x

    def route(self, x):
        return self.routing(self.rank, x.shape[0], self.E, self.k)

    def gather(self, x, rows):
        return x[rows.to(torch.int64)]

    def experts_forward(self, rows, ids, gates):
        assert ids.numel() == 0 or (int(ids.min()) >= 0 and int(ids.max()) < self.n_local)
        scale = (ids.to(torch.float64) + self.e0 + 1) * gates.to(torch.float64)
        return rows * scale.view(-1, 1)

    def shared_forward(self, x, sg):
        return x * (1000.0 * sg.to(torch.float64)).view(-1, 1)

    def combine(self, returned, pos, base):
        acc = base.clone()
        for j in range(pos.shape[1]):
            acc = acc + returned[pos[:, j].to(torch.int64)]
        return acc

    @classmethod
    def expected(cls, rank: int, T: int):
        x = cls.tokens(rank, T)
        idx, gates, sg = cls.routing(rank, T, cls.E, cls.k)
        s = ((idx.to(torch.float64) + 1) * gates.to(torch.float64)).sum(1) + 1000.0 * sg.to(torch.float64)
        return x * s.view(-1, 1)
