"""The allocation-free routing entry point (moe_route_static) against moe_route, through the C ABI.

moe_route_static serves callers that may not call cudaMalloc (e.g. while a CUDA graph is being
recorded, or inside a framework that owns all device memory): it keeps its scratch in a fixed
array inside the library.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_expert_router_b200 import _lib as M
from bit_grouped_expert_router_b200 import build as B
from bit_grouped_expert_router_b200 import synth
from helpers import gapped_x

pytestmark = pytest.mark.gpu


def _route_static(x, w, shape, T):
    idx = torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda")
    gates = torch.full((T, shape.k), -1.0, dtype=torch.float32, device="cuda")
    bias = w["router_bias"]
    rc = M.lib().moe_route_static(x.data_ptr(), T, shape.H, w["router"].data_ptr(),
                                  None if bias is None else bias.data_ptr(), shape.E, shape.k,
                                  idx.data_ptr(), gates.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    return rc, idx, gates


@pytest.mark.parametrize("name,T", [("decode", 16), ("prefill4k_zipf", 4)])
def test_route_static_matches_route_twice(name, T):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    shape = synth.WORKLOADS[name]
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol, T=T).cuda()
    wc = {n: (v.cuda() if v is not None else None) for n, v in w.items()}
    layer = M.Layer.from_shape(wc, shape, max_tokens=T, decode_max_tokens=T)
    ref = layer.route(x)
    for _ in range(2):                      # two calls in a row share the static scratch
        rc, idx, gates = _route_static(x, wc, shape, T)
        assert rc == M.MOE_OK, M.lib().moe_last_error()
        torch.cuda.synchronize()
        assert torch.equal(idx.cpu(), ref["idx"].cpu())
        np.testing.assert_allclose(gates.cpu().numpy(), ref["gates"].cpu().numpy(), rtol=1e-5, atol=2e-6)
    # beyond the static scratch: refused before launch, nothing written
    big = torch.zeros((shape.T * 0 + 64, shape.H), dtype=torch.bfloat16, device="cuda")
    rc, idx, _ = _route_static(big, wc, shape, 64)
    assert rc == M.MOE_ERR_TOO_LARGE
    assert "scratch" in M.lib().moe_last_error().decode()
    torch.cuda.synchronize()
    assert (idx.cpu() == -1).all()
    layer.close()
