"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point
include/moe.h declares, and rejects bad arguments before touching the device."""
import ctypes

import pytest
import torch

from bit_grouped_expert_router_b200 import _lib as M
from bit_grouped_expert_router_b200 import build as B


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.lib()


def test_exports_every_declared_symbol(lib):
    names = M.header_functions()
    assert set(names) >= {"moe_create", "moe_forward", "moe_forward_host", "moe_forward_host_async",
                          "moe_route", "moe_status",
                          "moe_debug_copy", "moe_device_bytes", "moe_last_error", "moe_destroy",
                          "moe_version"}
    for n in names:
        assert hasattr(lib, n), n


def test_version(lib):
    assert lib.moe_version() >= 10000


def _cfg(**kw):
    d = dict(H=2048, I=512, E=256, k=8, has_shared=True, max_tokens=4096, decode_max_tokens=16)
    d.update(kw)
    return M.make_config(d["H"], d["I"], d["E"], d["k"], d["has_shared"], d["max_tokens"],
                         d["decode_max_tokens"], d.get("flags", 0), d.get("group", 64))


def test_device_bytes_counts_the_repacked_layer(lib):
    n = lib.moe_device_bytes(ctypes.byref(_cfg()))
    per_expert = 3 * 512 * 2048 // 2 + 3 * 512 * 2048 // 64 * 4
    assert per_expert == 1769472
    assert n >= 257 * per_expert + 256 * 2048 * 4


@pytest.mark.parametrize("bad", [dict(group=32), dict(H=200), dict(I=96), dict(E=0), dict(E=300),
                                 dict(k=0), dict(k=33, E=64), dict(k=9, E=8), dict(max_tokens=0),
                                 dict(decode_max_tokens=-1), dict(decode_max_tokens=65536), dict(flags=0x80), dict(flags=0x200),
                                 dict(flags=0x60), dict(flags=0x50),
                                 dict(k=16, decode_max_tokens=2)])
def test_invalid_config_is_rejected_before_any_cuda_call(lib, bad):
    cfg = _cfg(**bad)
    assert lib.moe_device_bytes(ctypes.byref(cfg)) == 0
    h = ctypes.c_void_p()
    w = M.MoeWeights()
    rc = lib.moe_create(ctypes.byref(cfg), ctypes.byref(w), 0, None, ctypes.byref(h))
    assert rc == M.MOE_ERR_INVALID_ARG
    assert lib.moe_last_error().decode()
    assert h.value is None


def test_null_weights_rejected(lib):
    h = ctypes.c_void_p()
    rc = lib.moe_create(ctypes.byref(_cfg()), ctypes.byref(M.MoeWeights()), 0, None, ctypes.byref(h))
    assert rc == M.MOE_ERR_INVALID_ARG
    assert "weight" in lib.moe_last_error().decode()


def test_null_handle_calls(lib):
    assert lib.moe_forward(None, None, 1, None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_route(None, None, 1, None, None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_status(None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host(None, None, 1, None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host_async(None, None, 1, None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_copy(None, 0, None, 0, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_routed(None, None, 1, None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_rows(None, None, 0, None, 1, 1, None, None, None) == M.MOE_ERR_INVALID_ARG
    lib.moe_destroy(None)


def test_router_only_handle_owns_no_expert_weights(lib):
    full = lib.moe_device_bytes(ctypes.byref(_cfg()))
    router_only = lib.moe_device_bytes(ctypes.byref(_cfg(flags=M.MOE_FLAG_NO_EXPERTS)))
    per_expert = 1769472 * 257   # packed codes + fp16 scale/bias pairs of 256 experts + the shared one
    assert full - router_only >= per_expert
    assert lib.moe_device_bytes(ctypes.byref(_cfg(flags=M.MOE_FLAG_NO_ROUTER))) == full


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_router_only_create_needs_only_router_pointers(lib):
    # only the router pointers are checked before the device: NULL expert weights pass validation
    fake = ctypes.c_void_p(0x1000).value
    w = M.MoeWeights(router=fake, shared_gate=fake)
    h = ctypes.c_void_p()
    rc = lib.moe_create(ctypes.byref(_cfg(flags=M.MOE_FLAG_NO_EXPERTS)), ctypes.byref(w), 0, None, ctypes.byref(h))
    assert rc == M.MOE_ERR_CUDA, lib.moe_last_error().decode()
    w2 = M.MoeWeights(q_gate=fake)
    rc = lib.moe_create(ctypes.byref(_cfg(flags=M.MOE_FLAG_NO_EXPERTS)), ctypes.byref(w2), 0, None, ctypes.byref(h))
    assert rc == M.MOE_ERR_INVALID_ARG and "router" in lib.moe_last_error().decode()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_create_without_a_gpu_reports_cuda_error(lib):
    fake = ctypes.c_void_p(0x1000)  # aligned, never dereferenced: the device check fails first
    w = M.MoeWeights(*[fake.value] * len(M._WEIGHT_FIELDS))
    h = ctypes.c_void_p()
    rc = lib.moe_create(ctypes.byref(_cfg()), ctypes.byref(w), 0, None, ctypes.byref(h))
    assert rc in (M.MOE_ERR_CUDA, M.MOE_ERR_INVALID_ARG)
    assert lib.moe_last_error().decode()


def test_flush_to_zero_builds_are_refused():
    """The decode GEMVs carry 4-bit codes as fp32 subnormals; the build refuses flush-to-zero and
    fast-math flags, and its own flag list holds none of them."""
    for f in B.FORBIDDEN_FLAGS:
        assert f not in B.NVCC_FLAGS
        with pytest.raises(ValueError):
            B.check_flags(list(B.NVCC_FLAGS) + [f])
    B.check_flags(B.NVCC_FLAGS)


def test_subnormal_fmas_are_explicit_ptx():
    """Every FMA that multiplies a subnormal weight code is the explicit fma.rn.f32 helper, never
    fmaf (which -ftz=true would turn into a flushing instruction)."""
    import os
    import re
    csrc = os.path.join(os.path.dirname(B.__file__), "csrc")
    for name in os.listdir(csrc):
        if not name.endswith(".cu"):
            continue
        src = open(os.path.join(csrc, name)).read()
        assert not re.search(r"fmaf\(__uint_as_float\(__byte_perm", src), name
