"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Every step of the layer runs in the CUDA library; this module turns torch tensors into the
pointers and sizes the C ABI takes and turns return codes into exceptions.  There is no fallback:
if libmoe.so has not been built, loading fails loudly (run ``python -m
bit_grouped_expert_router_b200.build`` or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "moe.h")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_DEVICE = 2
MOE_ERR_TOO_LARGE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_DEVICE_BOUNDS = 6
MOE_ERR_RANGE = 7
MOE_FLAG_ROUTER_SIMT = 0x1
MOE_FLAG_DECODE_UNFUSED = 0x2
MOE_FLAG_POISON_WORKSPACE = 0x4
MOE_FLAG_HOST_SYNC_ROUTING = 0x8
MOE_FLAG_DEQUANT_TO_HBM = 0x10
MOE_FLAG_NO_ROUTER = 0x20
MOE_FLAG_NO_EXPERTS = 0x40
MOE_FLAG_TEST_STALL = 0x100

_ERR_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_DEVICE", 3: "TOO_LARGE", 4: "CUDA",
              5: "DEVICE_TIMEOUT", 6: "DEVICE_BOUNDS", 7: "RANGE"}


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libmoe {_ERR_NAMES.get(code, code)} ({code}): {msg}")
        self.code = code


class MoeConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("group", ctypes.c_int32), ("has_shared", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("decode_max_tokens", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


_WEIGHT_FIELDS = ["q_gate", "q_up", "q_down", "s_gate", "b_gate", "s_up", "b_up", "s_down", "b_down",
                  "qs_gate", "qs_up", "qs_down", "ss_gate", "bs_gate", "ss_up", "bs_up", "ss_down",
                  "bs_down", "router", "router_bias", "shared_gate"]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _WEIGHT_FIELDS]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (no rebuild, no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so not built at {LIB_PATH}; run bit_grouped_expert_router_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        L.moe_create.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), ctypes.c_int, P,
                                 ctypes.POINTER(P)]
        L.moe_forward.argtypes = [P, P, I32, P, P]
        L.moe_forward_host.argtypes = [P, P, I32, P, P]
        L.moe_forward_host_async.argtypes = [P, P, I32, P, P]
        L.moe_route.argtypes = [P, P, I32, P, P, P, P, P, P]
        L.moe_status.argtypes = [P]
        L.moe_debug_copy.argtypes = [P, ctypes.c_int, P, SZ, P]
        L.moe_device_bytes.argtypes = [ctypes.POINTER(MoeConfig)]
        L.moe_device_bytes.restype = SZ
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_destroy.argtypes = [P]
        L.moe_destroy.restype = None
        L.moe_version.restype = ctypes.c_int
        L.moe_profile_enable.argtypes = [P, ctypes.c_int]
        L.moe_profile_read.argtypes = [P, P, P]
        L.moe_route_static.argtypes = [P, I32, I32, P, P, I32, I32, P, P, P]
        L.moe_forward_routed.argtypes = [P, P, I32, P, P, P, P, P]
        L.moe_combine_rows.argtypes = [P, P, I32, P, I32, I32, P, P, P]
        for n in ("moe_create", "moe_forward", "moe_forward_host", "moe_forward_host_async", "moe_route", "moe_status",
                  "moe_debug_copy", "moe_profile_enable", "moe_profile_read", "moe_route_static",
                  "moe_forward_routed", "moe_combine_rows"):
            getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def header_functions():
    """Names of the functions include/moe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def check(code: int) -> None:
    if code != MOE_OK:
        raise MoeError(code, lib().moe_last_error().decode())


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def make_config(H, I, E, k, has_shared=True, max_tokens=4096, decode_max_tokens=16, flags=0,
                group=64) -> MoeConfig:
    return MoeConfig(H, I, E, k, group, 1 if has_shared else 0, max_tokens, decode_max_tokens, flags)


class Layer:
    """One MoE layer held by libmoe on a CUDA device.

    ``weights``: dict of CUDA tensors in the public layout (see include/moe.h; the names match the
    moe_weights fields).  The library repacks them into memory it owns, so they may be dropped
    after construction.
    """

    def __init__(self, weights: Dict[str, object], H: int, I: int, E: int, k: int, has_shared=True,
                 max_tokens: int = 4096, decode_max_tokens: int = 16, flags: int = 0, device=None,
                 stream=None):
        import torch
        self.H, self.I, self.E, self.k = H, I, E, k
        self.has_shared = bool(has_shared)
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        self.cfg = make_config(H, I, E, k, has_shared, max_tokens, decode_max_tokens, flags)
        w = MoeWeights(*[_ptr(weights.get(n)) for n in _WEIGHT_FIELDS])
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            check(lib().moe_create(ctypes.byref(self.cfg), ctypes.byref(w), self.device.index,
                                   _stream_ptr(stream), ctypes.byref(h)))
        self._h = h

    @classmethod
    def from_shape(cls, weights, shape, **kw):
        return cls(weights, shape.H, shape.I, shape.E, shape.k, shape.has_shared, **kw)

    @property
    def handle(self):
        if self._h is None:
            raise RuntimeError("layer has been closed")
        return self._h

    def forward(self, x, out=None, stream=None):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        check(lib().moe_forward(self.handle, _ptr(x), T, _ptr(out), _stream_ptr(stream)))
        return out

    def forward_host(self, x_host, out_host=None, stream=None):
        import torch
        T = x_host.shape[0]
        if out_host is None:
            out_host = torch.empty((T, self.H), dtype=torch.bfloat16, pin_memory=True)
        check(lib().moe_forward_host(self.handle, _ptr(x_host), T, _ptr(out_host), _stream_ptr(stream)))
        return out_host

    def forward_host_async(self, x_host, out_host, stream=None):
        """Enqueue copy-in, layer and copy-out on `stream` and return; `out_host` is valid once the
        stream has passed this call (pinned host tensors give overlapped copies)."""
        check(lib().moe_forward_host_async(self.handle, _ptr(x_host), x_host.shape[0], _ptr(out_host),
                                           _stream_ptr(stream)))
        return out_host

    def forward_routed(self, x, idx, gates, shared_gate=None, out=None, stream=None):
        """out[T, H] bf16 = sum_j gates[:, j] FFN_{idx[:, j]}(x) (+ shared_gate FFN_shared(x)) with the
        routing given: idx [T, k] int32, gates [T, k] fp32, shared_gate [T] fp32 (has_shared)."""
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        check(lib().moe_forward_routed(self.handle, _ptr(x), T, _ptr(idx), _ptr(gates), _ptr(shared_gate),
                                       _ptr(out), _stream_ptr(stream)))
        return out

    def combine_rows(self, rows, pos, base=None, out=None, stream=None):
        """out[T, H] bf16 = base + sum over j of rows[pos[:, j]] (pos < 0: no row), fp32 sums."""
        import torch
        T, k = pos.shape
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=pos.device)
        check(lib().moe_combine_rows(self.handle, _ptr(rows), rows.shape[0], _ptr(pos), T, k, _ptr(base),
                                     _ptr(out), _stream_ptr(stream)))
        return out

    def route(self, x, stream=None):
        """-> dict(idx [T,k] int32, gates [T,k] f32, shared_gate [T] f32, offsets [E+1] int32,
        perm [T*k] int32), all on the device."""
        import torch
        T = x.shape[0]
        dev = x.device
        r = dict(idx=torch.empty((T, self.k), dtype=torch.int32, device=dev),
                 gates=torch.empty((T, self.k), dtype=torch.float32, device=dev),
                 shared_gate=torch.empty(T, dtype=torch.float32, device=dev),
                 offsets=torch.empty(self.E + 1, dtype=torch.int32, device=dev),
                 perm=torch.empty(T * self.k, dtype=torch.int32, device=dev))
        check(lib().moe_route(self.handle, _ptr(x), T, _ptr(r["idx"]), _ptr(r["gates"]),
                              _ptr(r["shared_gate"]), _ptr(r["offsets"]), _ptr(r["perm"]),
                              _stream_ptr(stream)))
        return r

    def debug_copy(self, which: int, dst, stream=None):
        check(lib().moe_debug_copy(self.handle, which, _ptr(dst), dst.numel() * dst.element_size(),
                                   _stream_ptr(stream)))
        return dst

    PROF_SLOTS = ["router", "topk", "bucket_scan", "scatter", "gemm_gateup", "gemm_down", "finalize",
                  "gemv_gateup", "gemv_down", "decode_fused", "gather_rows"]

    def profile(self, enable: bool = True):
        check(lib().moe_profile_enable(self.handle, 1 if enable else 0))

    def profile_read(self):
        """-> {slot: (total_ms, launches)} for the calls recorded since profile(True)."""
        ms = (ctypes.c_float * len(self.PROF_SLOTS))()
        n = (ctypes.c_int32 * len(self.PROF_SLOTS))()
        check(lib().moe_profile_read(self.handle, ctypes.cast(ms, ctypes.c_void_p),
                                     ctypes.cast(n, ctypes.c_void_p)))
        return {s: (float(ms[i]), int(n[i])) for i, s in enumerate(self.PROF_SLOTS) if n[i]}

    def status(self) -> int:
        """Synchronise and return the device status code (MOE_OK or MOE_ERR_*); clears it."""
        return int(lib().moe_status(self.handle))

    def close(self):
        if getattr(self, "_h", None) is not None:
            lib().moe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
