"""Expert parallelism on CPU: the dispatch plan against brute force, and two gloo ranks running the
whole dispatch -> experts -> return -> combine flow (bit_grouped_expert_router_b200.ep) with exact
labelled rows and with the oracle's arithmetic."""
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_grouped_expert_router_b200.ep import Exchange, ExpertParallelLayer, plan_dispatch  # noqa: E402


@pytest.mark.parametrize("T,k,E,W", [(37, 8, 256, 4), (5, 2, 16, 2), (0, 3, 12, 3), (9, 4, 8, 1)])
def test_dispatch_plan_matches_brute_force(T, k, E, W):
    g = torch.Generator().manual_seed(T * 131 + k)
    idx = torch.randint(0, E, (T, k), generator=g, dtype=torch.int32)
    gates = torch.rand((T, k), generator=g)
    n = E // W
    p = plan_dispatch(idx, gates, n, W)
    # brute force: walk the pairs in (token, slot) order once per rank
    sent = [(t * k + j) for r in range(W) for t in range(T) for j in range(k) if int(idx[t, j]) // n == r]
    assert p.order.tolist() == sent
    assert p.send_counts.tolist() == [sum(1 for t in range(T) for j in range(k) if int(idx[t, j]) // n == r)
                                      for r in range(W)]
    for q, flat in enumerate(sent):
        t, j = divmod(flat, k)
        assert int(p.pair_token[q]) == t
        assert int(p.local_ids[q]) == int(idx[t, j]) - (int(idx[t, j]) // n) * n
        assert float(p.gates[q]) == float(gates[t, j])
        assert int(p.pos[t, j]) == q
    assert p.pos.shape == (T, k) and p.pos.dtype == torch.int32


def test_dispatch_plan_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        plan_dispatch(torch.tensor([[0, 16]], dtype=torch.int32), torch.ones(1, 2), 8, 2)


def test_one_rank_without_a_group_is_exact():
    sys.path.insert(0, os.path.dirname(__file__))
    from ep_shards import LabelShard
    layer = ExpertParallelLayer(LabelShard(0, 1), Exchange(None, 1))
    x = LabelShard.tokens(0, 11)
    assert torch.equal(layer.forward(x), LabelShard.expected(0, 11))


RANK_CODE = r"""
import os, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, os.path.join({root!r}, "tests"))
import datetime
import torch, torch.distributed as dist
from bit_grouped_expert_router_b200.ep import Exchange, ExpertParallelLayer
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
mode = {mode!r}
if mode == "labels":
    from ep_shards import LabelShard
    layer = ExpertParallelLayer(LabelShard(rank, world), Exchange(None if world == 1 else dist.group.WORLD, world))
    for T in (13, 0, 1, 40):     # ranks with different token counts in the same call
        T_r = T + 3 * rank if T else 0
        out = layer.forward(LabelShard.tokens(rank, T_r))
        assert torch.equal(out, LabelShard.expected(rank, T_r)), (T_r, out, LabelShard.expected(rank, T_r))
    print("LABELS OK", flush=True)
else:
    import numpy as np
    from bit_grouped_expert_router_b200 import synth
    from oracle import OracleLayer
    from ep_shards import OracleShard
    from parity import compare
    shape = synth.WORKLOADS["tiny"]
    w = synth.make_layer(shape, 0)
    ol = OracleLayer.from_shape(w, shape)
    layer = ExpertParallelLayer(OracleShard(ol, rank, world), Exchange(dist.group.WORLD, world))
    x = synth.make_x(shape, 0, chunk=rank, T=6 + 2 * rank)
    out = layer.forward(x)
    ref = ol.forward(x)
    compare(out, ref)
    print("ORACLE OK", flush=True)
dist.barrier()
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(mode, world=2):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", RANK_CODE.format(root=ROOT, mode=mode)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=240)
        finally:
            if p.poll() is None:
                p.kill()
        assert p.returncode == 0, err[-3000:]
        outs.append(out)
    return outs


def test_two_gloo_ranks_move_every_row_to_its_expert_and_back():
    for out in _run_ranks("labels"):
        assert "LABELS OK" in out


def test_two_gloo_ranks_match_the_single_process_oracle():
    for out in _run_ranks("oracle"):
        assert "ORACLE OK" in out
