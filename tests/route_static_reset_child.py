"""Child process of tests/test_zz_no_alloc.py: moe_route_static across a reset of the CUDA context.

Runs without torch's CUDA state: buffers are allocated and copied with the CUDA driver API (via
ctypes), so resetting the device's primary context leaves nothing of this process dangling.  The
call is made once, the primary context is reset (all of its allocations and loaded modules are
destroyed), a new context is made current, and the call is made again with fresh buffers.  The
library must find its static scratch array in the new context; both calls are checked against
the oracle.  Prints one line "ok ..." or "skip ..." and exits 0, or raises.
"""
import ctypes
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from bit_grouped_expert_router_b200 import _lib as M  # noqa: E402
from bit_grouped_expert_router_b200 import synth  # noqa: E402
from helpers import gapped_x  # noqa: E402

cu = ctypes.CDLL("libcuda.so.1")


def ck(r, what):
    if r != 0:
        raise RuntimeError(f"{what}: CUresult {r}")


def make_current(dev):
    ctx = ctypes.c_void_p()
    ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(ctx), dev), "cuDevicePrimaryCtxRetain")
    ck(cu.cuCtxSetCurrent(ctx), "cuCtxSetCurrent")
    cid = ctypes.c_ulonglong()
    ck(cu.cuCtxGetId(ctx, ctypes.byref(cid)), "cuCtxGetId")
    return cid.value


def upload(a):
    a = np.ascontiguousarray(a)
    p = ctypes.c_uint64()
    ck(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(max(a.nbytes, 16))), "cuMemAlloc")
    ck(cu.cuMemcpyHtoD_v2(p, a.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(a.nbytes)), "cuMemcpyHtoD")
    return p.value


def download(p, shape, dtype):
    out = np.empty(shape, dtype)
    ck(cu.cuMemcpyDtoH_v2(out.ctypes.data_as(ctypes.c_void_p), ctypes.c_uint64(p), ctypes.c_size_t(out.nbytes)),
       "cuMemcpyDtoH")
    return out


def one_call(x_bits, router, shape, T, ref_idx, ref_g):
    px, pr = upload(x_bits), upload(router)
    pidx = upload(np.full((T, shape.k), -1, np.int32))
    pg = upload(np.full((T, shape.k), -1, np.float32))
    rc = M.lib().moe_route_static(px, T, shape.H, pr, None, shape.E, shape.k, pidx, pg, None)
    if rc != M.MOE_OK:
        raise RuntimeError(f"moe_route_static: {rc} {M.lib().moe_last_error().decode()}")
    ck(cu.cuCtxSynchronize(), "cuCtxSynchronize")
    idx = download(pidx, (T, shape.k), np.int32)
    g = download(pg, (T, shape.k), np.float32)
    assert (idx == ref_idx).all(), "expert indices differ from the oracle"
    np.testing.assert_allclose(g, ref_g, rtol=1e-5, atol=2e-6)


def main():
    shape = synth.WORKLOADS["decode"]
    T = 8
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol, T=T)
    ref_idx, ref_g, _, _ = ol.route(x)
    x_bits = x.view(__import__("torch").int16).numpy().view(np.uint16)
    router = w["router"].numpy().astype(np.float32)

    ck(cu.cuInit(0), "cuInit")
    dev = ctypes.c_int()
    ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
    id0 = make_current(dev)
    one_call(x_bits, router, shape, T, ref_idx, ref_g)
    ck(cu.cuDevicePrimaryCtxReset_v2(dev), "cuDevicePrimaryCtxReset")
    id1 = make_current(dev)
    if id1 == id0:
        # the library keys its cached address on this id; a reused id would make the second call
        # use the old address, so it is not made
        print(f"skip: the driver kept context id {id0} across the reset")
        return
    one_call(x_bits, router, shape, T, ref_idx, ref_g)
    print(f"ok: context {id0} -> {id1}, both calls match the oracle")


if __name__ == "__main__":
    main()
