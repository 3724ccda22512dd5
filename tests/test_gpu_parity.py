"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Expert indices, bucket offsets and the bucket permutation must match the oracle bit for bit (the
activations are drawn so the top-(k+1) fp64 logits of every token are >= 1e-3 apart); gates to
fp32 accuracy; layer outputs within the tolerance in tests/parity.py.  Sizes: the tiny layer and
small ragged shapes span several tiles and a ragged tail; the full workloads (T = 1, 512, 4096)
are compared on every token's routing and on all (T <= 512) or a seeded sample of 256 tokens'
outputs, in the same launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_expert_router_b200 import _lib as M
from bit_grouped_expert_router_b200 import build as B
from bit_grouped_expert_router_b200 import synth
from helpers import gapped_x
from parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    M.lib()


def _cuda(w):
    return {k: (v.cuda() if v is not None else None) for k, v in w.items()}


def _layer(w, shape, **kw):
    return M.Layer.from_shape(_cuda(w), shape, **kw)


def _route_check(layer, ol, x, shape):
    r = layer.route(x.cuda())
    torch.cuda.synchronize()
    idx, g, sg, _ = ol.route(x)
    assert (r["idx"].cpu().numpy() == idx).all(), "expert indices differ"
    np.testing.assert_allclose(r["gates"].cpu().numpy(), g, rtol=1e-5, atol=2e-6)
    if shape.has_shared:
        np.testing.assert_allclose(r["shared_gate"].cpu().numpy(), sg, rtol=1e-5, atol=2e-6)
    _, off, perm = oracle.bucket(idx, shape.E)
    assert (r["offsets"].cpu().numpy() == off).all(), "bucket offsets differ"
    assert (r["perm"].cpu().numpy() == perm).all(), "bucket permutation differs"
    assert layer.status() == M.MOE_OK


def _forward_check(layer, ol, x, tokens=None):
    out = layer.forward(x.cuda())
    torch.cuda.synchronize()
    assert layer.status() == M.MOE_OK
    ref = ol.forward(x, tokens=tokens)
    got = out.cpu() if tokens is None else out.cpu()[torch.as_tensor(tokens, dtype=torch.long)]
    return compare(got, ref)


# ---------------------------------------------------------------------------------------------
# tiny layer and small ragged shapes: both paths, every token
TINY = synth.WORKLOADS["tiny"]
RAGGED = synth.Shape("ragged", T=300, H=512, E=32, k=4, I=256, zipf_s=1.1, seed=21)
NOSHARED = synth.Shape("noshared", T=77, H=256, E=16, k=2, I=128, has_shared=False, seed=22)
KEQE = synth.Shape("k_eq_e", T=40, H=256, E=8, k=8, I=128, seed=23)
SINGLE = synth.Shape("single", T=130, H=256, E=1, k=1, I=192, has_shared=False, seed=24)


@pytest.mark.parametrize("shape", [TINY, RAGGED, NOSHARED, KEQE, SINGLE], ids=lambda s: s.name)
@pytest.mark.parametrize("path", ["prefill", "decode"])
def test_small_shapes(shape, path):
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    dec = 0 if path == "prefill" else shape.T
    layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=dec)
    _route_check(layer, ol, x, shape)
    _forward_check(layer, ol, x)
    # every prefix length exercises ragged tiles: 1, a tile boundary +/- 1 and the whole
    for T in sorted({1, 2, min(shape.T, 17), min(shape.T, 128), min(shape.T, 129), shape.T}):
        _forward_check(layer, ol, x[:T])
    layer.close()


BIGK = synth.Shape("big_k", T=70, H=256, E=64, k=24, I=128, seed=25)


def test_many_experts_per_token():
    """k = 24: the first 64-token bucketing block holds 1536 routed entries, which the scatter ranks
    in two rounds of 1024, and the second block is ragged (6 tokens); indices, offsets and the
    permutation bit-exact, outputs within tolerance (prefill path)."""
    w = synth.make_layer(BIGK)
    ol = oracle.OracleLayer.from_shape(w, BIGK)
    x = gapped_x(BIGK, ol)
    layer = _layer(w, BIGK, max_tokens=BIGK.T, decode_max_tokens=0)
    _route_check(layer, ol, x, BIGK)
    _forward_check(layer, ol, x)
    _forward_check(layer, ol, x[:65])
    layer.close()


@pytest.mark.parametrize("shape", [TINY, RAGGED], ids=lambda s: s.name)
def test_poisoned_workspace_changes_no_result(shape):
    """Sanitiser substitute: the workspace starts as 0xFF bytes (NaN / -1) instead of zeros, so a
    kernel that reads workspace it did not write first would give non-finite or wrong outputs.
    Both paths (prefill; batch-1 fused decode; multi-token GEMV decode) still match the oracle."""
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    for dec in (0, shape.T):
        layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=dec, flags=M.MOE_FLAG_POISON_WORKSPACE)
        _route_check(layer, ol, x, shape)
        for T in sorted({1, 2, min(shape.T, 129), shape.T}):
            _forward_check(layer, ol, x[:T])
        layer.close()


@pytest.mark.parametrize("shape", [TINY, RAGGED], ids=lambda s: s.name)
def test_host_synchronised_routing_ablation_changes_no_result(shape):
    """The ablation flag only moves a host round trip between routing and the grouped GEMMs."""
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=0, flags=M.MOE_FLAG_HOST_SYNC_ROUTING)
    for T in sorted({2, min(shape.T, 129), shape.T}):
        _forward_check(layer, ol, x[:T])
    layer.close()


@pytest.mark.parametrize("shape", [TINY, RAGGED], ids=lambda s: s.name)
def test_fp16_weights_in_hbm_ablation_matches_the_oracle(shape):
    """The ablation variant (A tiles dequantised once to fp16 in HBM, loaded by TMA) computes the
    same layer: both grouped-GEMM launch shapes (T * k below and above 64 * E)."""
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=0, flags=M.MOE_FLAG_DEQUANT_TO_HBM)
    for T in sorted({2, min(shape.T, 129), shape.T}):
        _forward_check(layer, ol, x[:T])
    layer.close()


def test_tiny_intermediate_activations_match():
    """The gate/up GEMM alone: act rows in bucket order vs silu(Wg x) * (Wu x) from the oracle's
    dequantised weights (fp64), within fp16 rounding."""
    shape = TINY
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=0)
    layer.forward(x.cuda())
    rows = shape.T * shape.k + shape.T
    act = torch.empty((rows, shape.I), dtype=torch.float16, device="cuda")
    layer.debug_copy(0, act)
    torch.cuda.synchronize()
    idx, _, _, _ = ol.route(x)
    _, _, perm = oracle.bucket(idx, shape.E)
    X = x.float().double().numpy()
    for p in range(rows):
        if p < shape.T * shape.k:
            t, e = perm[p] // shape.k, idx.ravel()[perm[p]]
            sfx, ee = "", e
        else:
            t, sfx, ee = p - shape.T * shape.k, "s", None
        def dq(n):
            q, s, b = w["q" + sfx + "_" + n], w["s" + sfx + "_" + n], w["b" + sfx + "_" + n]
            if ee is not None:
                q, s, b = q[ee], s[ee], b[ee]
            return oracle.dequant(q, s, b, shape.I, shape.H).astype(np.float64)
        gz = dq("gate") @ X[t]
        ref = gz / (1 + np.exp(-gz)) * (dq("up") @ X[t])
        got = act[p].float().double().cpu().numpy()
        np.testing.assert_allclose(got, ref, rtol=2e-3, atol=2e-3)
    layer.close()


# ---------------------------------------------------------------------------------------------
# full-size workloads in the benchmark's launch configuration
def _full(name, layer_idx=0, chunk=0, T=None):
    shape = synth.WORKLOADS[name]
    w = synth.make_layer(shape, layer_idx)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol, layer_idx, chunk, T)
    return shape, w, ol, x


def _sample(T, n, seed):
    if T <= n:
        return None
    return sorted(np.random.default_rng(seed).choice(T, n, replace=False).tolist())


@pytest.mark.parametrize("name,layer_idx,chunk", [("prefill512", 0, 0), ("prefill4k_zipf", 0, 0),
                                                  ("prefill16k_zipf", 0, 0), ("prefill16k_zipf", 39, 3)])
def test_full_prefill_workloads(name, layer_idx, chunk):
    shape, w, ol, x = _full(name, layer_idx, chunk)
    layer = _layer(w, shape, max_tokens=4096, decode_max_tokens=16)
    _route_check(layer, ol, x, shape)
    stats = _forward_check(layer, ol, x, tokens=_sample(shape.T, 256, 7 + layer_idx))
    print(name, stats)
    layer.close()


def test_one_16k_token_call_at_the_largest_sizes():
    """All 16384 tokens of a prompt in one call (max_tokens = 16384): the largest buckets (the
    skewed routing sends ~16k rows to its hottest expert), the longest tile list and the biggest
    workspace.  Routing and bucketing checked for every token, outputs on 256 sampled tokens."""
    shape = synth.shape_with(synth.WORKLOADS["prefill16k_zipf"], T=16384)
    w = synth.make_layer(shape, 0)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol, 0, 0)
    layer = _layer(w, shape, max_tokens=16384, decode_max_tokens=16)
    _route_check(layer, ol, x, shape)
    print("16k in one call", _forward_check(layer, ol, x, tokens=_sample(shape.T, 256, 11)))
    layer.close()


@pytest.mark.parametrize("layer_idx", [0, 39])
def test_full_decode_workload(layer_idx):
    shape, w, ol, x = _full("decode", layer_idx, 0, T=16)
    layer = _layer(w, shape, max_tokens=4096, decode_max_tokens=16)
    _route_check(layer, ol, x[:1], shape)
    print("decode T=1", _forward_check(layer, ol, x[:1]))
    print("decode T=2 (fused kernel, several tokens)", _forward_check(layer, ol, x[:2]))
    print("decode T=4 (fused kernel, several tokens)", _forward_check(layer, ol, x[:4]))
    print("decode T=5 (fused kernel, several tokens)", _forward_check(layer, ol, x[:5]))
    print("decode T=8 (fused kernel, several tokens)", _forward_check(layer, ol, x[:8]))
    print("decode T=9 (fused kernel, 8 + 1 tokens)", _forward_check(layer, ol, x[:9]))
    print("decode T=16 (fused kernel, 8 + 8 tokens)", _forward_check(layer, ol, x))
    # the multi-kernel GEMV chain, which serves shapes the fused kernel does not fit
    chain = _layer(w, shape, max_tokens=4096, decode_max_tokens=16, flags=M.MOE_FLAG_DECODE_UNFUSED)
    for T in (1, 2, 9, 16):
        print(f"decode T={T} (GEMV chain)", _forward_check(chain, ol, x[:T]))
    chain.close()
    # the same tokens through the prefill path agree too
    layer2 = _layer(w, shape, max_tokens=4096, decode_max_tokens=0)
    print("prefill T=16", _forward_check(layer2, ol, x))
    layer.close()
    layer2.close()


def test_both_grouped_gemm_launch_shapes_around_the_switch():
    """The grouped GEMMs run as two CTAs per SM with 128-token tiles while T * k <= 64 * E and as
    one CTA per SM with 256-token tiles above: T = 2048 and 2049 at the full layer sizes sit on
    either side of the switch (same layer, same leading tokens)."""
    shape = synth.Shape("switch", T=2049, H=2048, E=256, k=8, I=512, zipf_s=1.1, seed=32)
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=16)
    for T in (2048, 2049):
        sub = synth.shape_with(shape, T=T)
        _route_check(layer, ol, x[:T], sub)
        print("T =", T, _forward_check(layer, ol, x[:T], tokens=_sample(T, 96, 5)))
    layer.close()


def test_forced_experts_make_large_buckets():
    shape = synth.Shape("forced", T=1024, H=2048, E=256, k=8, I=512, seed=31)
    w = synth.make_layer(shape)
    chosen = [3, 40, 77, 100, 150, 201, 222, 255]
    bias = torch.zeros(shape.E)
    bias[chosen] = 100.0
    w["router_bias"] = bias
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    layer = _layer(w, shape, max_tokens=1024, decode_max_tokens=0)
    _route_check(layer, ol, x, shape)
    _forward_check(layer, ol, x, tokens=_sample(shape.T, 64, 3))
    layer.close()


# ---------------------------------------------------------------------------------------------
# boundary behaviour through the C ABI
def test_host_buffers_and_edge_calls():
    shape = TINY
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=2)
    dev = layer.forward(x.cuda()).cpu()
    host = layer.forward_host(x.pin_memory())
    assert torch.equal(dev.view(torch.int16), host.view(torch.int16))
    # the asynchronous variant: two handles on two streams, calls enqueued back to back
    layer2 = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=2)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    xh = x.pin_memory()
    outs = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    for _ in range(3):
        layer.forward_host_async(xh, outs[0], streams[0])
        layer2.forward_host_async(xh, outs[1], streams[1])
    for s in streams:
        s.synchronize()
    for o in outs:   # same inputs and weights: equal up to the order of the fp32 reductions
        torch.testing.assert_close(o.float(), dev.float(), rtol=1e-2, atol=1e-2)
    assert layer2.status() == M.MOE_OK
    layer2.close()
    # T = 0 is a no-op, T > max_tokens is refused before launch
    assert M.lib().moe_forward(layer.handle, x.cuda().data_ptr(), 0, None, None) == M.MOE_OK
    out = torch.empty((shape.T + 1, shape.H), dtype=torch.bfloat16, device="cuda")
    xx = torch.zeros((shape.T + 1, shape.H), dtype=torch.bfloat16, device="cuda")
    rc = M.lib().moe_forward(layer.handle, xx.data_ptr(), shape.T + 1, out.data_ptr(), None)
    assert rc == M.MOE_ERR_TOO_LARGE
    # misaligned pointer
    rc = M.lib().moe_forward(layer.handle, xx.data_ptr() + 2, 1, out.data_ptr(), None)
    assert rc == M.MOE_ERR_INVALID_ARG
    assert layer.status() == M.MOE_OK
    layer.close()


def test_fp16_range_overflow_is_reported():
    shape = synth.shape_with(TINY, T=4)
    w = synth.make_layer(shape)
    layer = _layer(w, shape, max_tokens=4, decode_max_tokens=0)
    x = torch.zeros((4, shape.H), dtype=torch.bfloat16)
    x[1, 5] = 1.0e6   # representable in bf16, not in fp16
    layer.forward(x.cuda())
    assert layer.status() == M.MOE_ERR_RANGE
    assert layer.status() == M.MOE_OK   # cleared
    layer.close()


# ---------------------------------------------------------------------------------------------
# batch-1 decode: the single cooperative kernel, the multi-kernel chain, and graph replay
def test_decode_fused_and_unfused_agree_and_replay_in_a_graph():
    shape = synth.WORKLOADS["decode"]
    layers, xs, refs = [], [], []
    for l in (0, 1):
        w = synth.make_layer(shape, l)
        ol = oracle.OracleLayer.from_shape(w, shape)
        x = gapped_x(shape, ol, l, 0, T=1)
        refs.append(ol.forward(x))
        xs.append(x.cuda())
        wc = _cuda(w)
        layers.append((M.Layer.from_shape(wc, shape, max_tokens=16, decode_max_tokens=16),
                       M.Layer.from_shape(wc, shape, max_tokens=16, decode_max_tokens=16,
                                          flags=M.MOE_FLAG_DECODE_UNFUSED)))
    for (fused, unfused), x, ref in zip(layers, xs, refs):
        a = fused.forward(x)
        b = unfused.forward(x)
        torch.cuda.synchronize()
        assert fused.status() == M.MOE_OK and unfused.status() == M.MOE_OK
        compare(a.cpu(), ref)
        compare(b.cpu(), ref)
        # repeated calls reuse the self-cleaning accumulator state
        for _ in range(3):
            a2 = fused.forward(x)
        torch.cuda.synchronize()
        compare(a2.cpu(), ref)
    # the fused kernels of two layers captured in one CUDA graph and replayed
    outs = [torch.empty((1, shape.H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for (fused, _), x, o in zip(layers, xs, outs):
            fused.forward(x, out=o)
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    for o, ref in zip(outs, refs):
        compare(o.cpu(), ref)
    del g
    for f, u in layers:
        assert f.status() == M.MOE_OK
        f.close()
        u.close()


# ---------------------------------------------------------------------------------------------
# failure detection without a GPU fault
def test_stalled_wait_times_out_and_the_context_stays_usable():
    """A bounded device-side wait that runs out.  With the test-only stall flag the prefill
    producer withholds every load, so the grouped GEMMs' consumer waits reach their limit: the
    kernels unwind and return, the status word reads MOE_ERR_DEVICE_TIMEOUT, and afterwards a
    normal layer on the same device computes correct results (the context was never lost)."""
    shape = TINY
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    stalled = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=0, flags=M.MOE_FLAG_TEST_STALL)
    stalled.forward(x.cuda())
    torch.cuda.synchronize()
    assert stalled.status() == M.MOE_ERR_DEVICE_TIMEOUT
    assert stalled.status() == M.MOE_OK   # reading the status clears it
    stalled.close()
    layer = _layer(w, shape, max_tokens=shape.T, decode_max_tokens=0)
    _forward_check(layer, ol, x)
    layer.close()


def test_decode_call_after_a_timed_out_one_is_correct():
    """Batch-1 decode: with the test-only stall flag the fused kernel withholds one router result
    on the handle's first call, so the routed units' bounded waits run out (about 1 s) and the call
    gives up part-way, leaving partial sums in the workspace.  The very next call -- made without
    reading the status in between -- must reset that state on the device and compute the right
    output; the status then reports the first call's timeout once."""
    shape = TINY
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol, T=1)
    ref = ol.forward(x)
    layer = _layer(w, shape, max_tokens=1, decode_max_tokens=1, flags=M.MOE_FLAG_TEST_STALL)
    xc = x.cuda()
    layer.forward(xc)                    # gives up part-way
    out = layer.forward(xc)              # no status read in between
    torch.cuda.synchronize()
    compare(out.cpu(), ref)
    assert layer.status() == M.MOE_ERR_DEVICE_TIMEOUT
    assert layer.status() == M.MOE_OK
    for _ in range(2):
        out = layer.forward(xc)
    torch.cuda.synchronize()
    compare(out.cpu(), ref)
    assert layer.status() == M.MOE_OK
    layer.close()
