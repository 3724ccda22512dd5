"""GPU parity of the routing-supplied forward (moe_forward_routed), the row combine
(moe_combine_rows) and the expert-parallel layer built on them (bit_grouped_expert_router_b200.ep)."""
import sys
import threading

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_expert_router_b200 import _lib as M
from bit_grouped_expert_router_b200 import build as B
from bit_grouped_expert_router_b200 import synth
from bit_grouped_expert_router_b200.ep import Exchange, ExpertParallelLayer, LibraryShard
from helpers import gapped_x
from parity import compare, ulp_bf16

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
RAGGED = synth.Shape("ragged", T=300, H=512, E=32, k=4, I=256, zipf_s=1.1, seed=21)
NOSHARED = synth.Shape("noshared", T=77, H=256, E=16, k=2, I=128, has_shared=False, seed=22)


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    M.lib()


def _cuda(w):
    return {k: (v.cuda() if v is not None else None) for k, v in w.items()}


def _setup(shape, T=None):
    w = synth.make_layer(shape, 0)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol, 0, 0, T)
    return w, ol, x


@pytest.mark.parametrize("shape,T", [(RAGGED, None), (NOSHARED, None), (RAGGED, 7), (TINY, 3)],
                         ids=["ragged-prefill", "noshared-prefill", "ragged-decode", "tiny-decode"])
def test_routed_forward_with_the_layers_own_routing_equals_forward(shape, T):
    w, ol, x = _setup(shape, T)
    layer = M.Layer.from_shape(_cuda(w), shape, max_tokens=512, decode_max_tokens=16,
                               flags=M.MOE_FLAG_DECODE_UNFUSED)
    xd = x.cuda()
    r = layer.route(xd)
    sg = r["shared_gate"] if shape.has_shared else None
    got = layer.forward_routed(xd, r["idx"], r["gates"], sg)
    want = layer.forward(xd)
    torch.cuda.synchronize()
    assert layer.status() == M.MOE_OK
    # the same kernels after the routing step; the combine's fp32 atomic sums may land in another
    # order, so the two agree to one bf16 rounding step, and both match the oracle
    g64, w64 = got.cpu().double().numpy(), want.cpu().double().numpy()
    assert (np.abs(g64 - w64) <= ulp_bf16(np.maximum(np.abs(g64), np.abs(w64)))).all()
    compare(got.cpu(), ol.forward(x))
    layer.close()


def _oracle_routed(ol, x, idx, gates, sg):
    xs = x.to(torch.float64).numpy()
    out = np.zeros((x.shape[0], ol.H))
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            out[t] += float(gates[t, j]) * ol.expert_ffn(int(idx[t, j]), xs[t])
        if sg is not None:
            out[t] += float(sg[t]) * ol.expert_ffn(ol.E, xs[t])
    return out


@pytest.mark.parametrize("shape,T", [(TINY, 40), (TINY, 5), (NOSHARED, 33)], ids=["prefill", "decode", "noshared"])
def test_routed_forward_with_arbitrary_routing_matches_the_oracle(shape, T):
    """Repeated experts within a token, negative and zero gates, gates not summing to one."""
    w, ol, x = _setup(shape, T)
    g = torch.Generator().manual_seed(5)
    idx = torch.randint(0, shape.E, (T, shape.k), generator=g, dtype=torch.int32)
    idx[0, :] = idx[0, 0]
    gates = (torch.rand((T, shape.k), generator=g) * 2 - 0.5).to(torch.float32)
    gates[1, :] = 0
    sg = torch.rand(T, generator=g).to(torch.float32) if shape.has_shared else None
    layer = M.Layer.from_shape(_cuda(w), shape, max_tokens=64, decode_max_tokens=8)
    got = layer.forward_routed(x.cuda(), idx.cuda(), gates.cuda(), sg.cuda() if sg is not None else None)
    torch.cuda.synchronize()
    assert layer.status() == M.MOE_OK
    compare(got.cpu(), _oracle_routed(ol, x, idx, gates, sg))
    layer.close()


def test_routed_forward_reports_an_out_of_range_expert_and_stays_usable():
    w, ol, x = _setup(TINY, 24)
    layer = M.Layer.from_shape(_cuda(w), TINY, max_tokens=64, decode_max_tokens=0)
    idx = torch.zeros((24, TINY.k), dtype=torch.int32)
    idx[3, 1] = TINY.E
    gates = torch.full((24, TINY.k), 0.5)
    sg = torch.full((24,), 0.5)
    layer.forward_routed(x.cuda(), idx.cuda(), gates.cuda(), sg.cuda())
    assert layer.status() == M.MOE_ERR_DEVICE_BOUNDS
    idx[3, 1] = 1
    got = layer.forward_routed(x.cuda(), idx.cuda(), gates.cuda(), sg.cuda())
    torch.cuda.synchronize()
    assert layer.status() == M.MOE_OK
    compare(got.cpu(), _oracle_routed(ol, x, idx, gates, sg))
    layer.close()


def test_combine_rows_is_the_fp32_sum_in_slot_order():
    w, ol, x = _setup(TINY, 8)
    layer = M.Layer.from_shape(_cuda(w), TINY, max_tokens=64)
    g = torch.Generator().manual_seed(9)
    T, k, n, H = 45, 5, 70, TINY.H
    rows = torch.randn((n, H), generator=g).to(torch.bfloat16)
    base = torch.randn((T, H), generator=g).to(torch.bfloat16)
    pos = torch.randint(-1, n, (T, k), generator=g, dtype=torch.int32)
    for b in (base, None):
        want = b.float() if b is not None else torch.zeros((T, H))
        for j in range(k):
            p = pos[:, j].to(torch.int64)
            want = want + torch.where((p >= 0).view(-1, 1), rows[p.clamp(min=0)].float(), torch.zeros(()))
        got = layer.combine_rows(rows.cuda(), pos.cuda(), base=b.cuda() if b is not None else None)
        torch.cuda.synchronize()
        assert torch.equal(got.cpu(), want.to(torch.bfloat16))
    bad = pos.clone()
    bad[2, 3] = n
    layer.combine_rows(rows.cuda(), bad.cuda())
    assert layer.status() == M.MOE_ERR_DEVICE_BOUNDS
    layer.close()


class ThreadExchange(Exchange):
    """All-to-all between shards run as threads of one process on one GPU: every exchange is a
    host-side hand-off of device tensors between two barriers (no kernel waits on another)."""

    def __init__(self, rank, world, board, barrier):
        super().__init__(None, world)
        self.rank, self.board, self.barrier = rank, board, barrier

    def _swap(self, parts):
        self.board[self.rank] = parts
        self.barrier.wait()
        got = [self.board[r][self.rank] for r in range(self.world)]
        self.barrier.wait()
        return got

    def counts(self, send_counts):
        return torch.stack(self._swap(list(send_counts.unbind(0))))

    def rows(self, send, send_splits, recv_splits, out=None):
        got = self._swap(list(torch.split(send, list(send_splits))))
        return torch.cat(got, 0) if got else send[:0]


def _ep_run(shape, w, xs, world):
    """EP forward of xs[r] on shard r of `world`, all shards in threads; -> list of outputs."""
    wd = _cuda(w)
    board, barrier = {}, threading.Barrier(world)
    shards = [LibraryShard(wd, shape.H, shape.I, shape.E, shape.k, shape.has_shared, r, world, max_tokens=512)
              for r in range(world)]
    outs, errs = [None] * world, []

    def run(r):
        try:
            layer = ExpertParallelLayer(shards[r], ThreadExchange(r, world, board, barrier))
            outs[r] = layer.forward(xs[r].cuda())
            torch.cuda.synchronize()
        except BaseException as e:   # surface a failure in the main thread, free the others
            errs.append(e)
            barrier.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    for s in shards:
        for L in (s.router, s.experts, s.shared):
            if L is not None:
                assert L.status() == M.MOE_OK
        s.close()
    if errs:
        raise errs[0]
    return outs


@pytest.mark.parametrize("shape", [RAGGED, NOSHARED], ids=lambda s: s.name)
def test_expert_parallel_one_rank_matches_the_oracle_and_forward(shape):
    w, ol, x = _setup(shape)
    (out,) = _ep_run(shape, w, [x], 1)
    compare(out.cpu(), ol.forward(x))
    layer = M.Layer.from_shape(_cuda(w), shape, max_tokens=512)
    ref = layer.forward(x.cuda()).cpu()
    layer.close()
    # the same experts per row, each gated term rounded to bf16 before the fp32 sum instead of
    # summed in fp32 first: within the output tolerance of the single-GPU forward too
    compare(out.cpu(), ref.double().numpy())


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_shards_equal_one_rank_over_all_tokens(world):
    """Each row's expert result does not depend on which shard or tile computes it, so W shards on
    their own token slices give the one-rank result over the concatenated tokens, bit for bit."""
    shape = RAGGED
    w, ol, x = _setup(shape)
    cuts = [0, 40, 41, 190, 300][: world] + [300]
    xs = [x[cuts[r]:cuts[r + 1]].contiguous() for r in range(world)]
    parts = _ep_run(shape, w, xs, world)
    (whole,) = _ep_run(shape, w, [x], 1)
    assert torch.equal(torch.cat([p.cpu() for p in parts], 0), whole.cpu())
    compare(torch.cat([p.cpu() for p in parts], 0), ol.forward(x))
