"""The allocation-free routing entry point (moe_route_static), through the C ABI.

moe_route_static serves callers that may not call cudaMalloc (e.g. while a CUDA graph is being
recorded, or inside a framework that owns all device memory): it keeps its scratch in a fixed
array inside the library.  Its results are checked against the oracle (expert indices bit for
bit, gates to fp32 accuracy) and against moe_route, on two calls in a row; free device memory
does not change across the calls; and a reset of the CUDA context between two calls (in a child
process that owns no torch CUDA state) leaves it working.  This file is collected last so that a
run stopping at the first failure has already run every other test; it also passes on its own in
a fresh process.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_expert_router_b200 import _lib as M
from bit_grouped_expert_router_b200 import build as B
from bit_grouped_expert_router_b200 import synth
from helpers import gapped_x

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


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
def test_route_static_matches_oracle_and_route_twice(name, T):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    shape = synth.WORKLOADS[name]
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x_host = gapped_x(shape, ol, T=T)
    ref_idx, ref_g, _, _ = ol.route(x_host)
    x = x_host.cuda()
    wc = {n: (v.cuda() if v is not None else None) for n, v in w.items()}
    layer = M.Layer.from_shape(wc, shape, max_tokens=T, decode_max_tokens=T)
    ref = layer.route(x)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):                      # two calls in a row share the static scratch
        rc, idx, gates = _route_static(x, wc, shape, T)
        assert rc == M.MOE_OK, M.lib().moe_last_error()
        torch.cuda.synchronize()
        assert (idx.cpu().numpy() == ref_idx).all(), "expert indices differ from the oracle"
        np.testing.assert_allclose(gates.cpu().numpy(), ref_g, rtol=1e-5, atol=2e-6)
        assert torch.equal(idx.cpu(), ref["idx"].cpu())
        np.testing.assert_allclose(gates.cpu().numpy(), ref["gates"].cpu().numpy(), rtol=1e-5, atol=2e-6)
    assert torch.cuda.mem_get_info()[0] == free0, "device memory changed across the calls"
    # beyond the static scratch: refused before launch, nothing written
    big = torch.zeros((64, shape.H), dtype=torch.bfloat16, device="cuda")
    rc, idx, _ = _route_static(big, wc, shape, 64)
    assert rc == M.MOE_ERR_TOO_LARGE
    assert "scratch" in M.lib().moe_last_error().decode()
    torch.cuda.synchronize()
    assert (idx.cpu() == -1).all()
    layer.close()


def test_route_static_after_a_context_reset():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES=os.environ.get("CUDA_VISIBLE_DEVICES", str(torch.cuda.current_device())))
    r = subprocess.run([sys.executable, os.path.join(HERE, "route_static_reset_child.py")], capture_output=True,
                       text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    last = r.stdout.strip().splitlines()[-1]
    if last.startswith("skip"):
        pytest.skip(last)
    assert last.startswith("ok"), r.stdout
