"""TEST INFRASTRUCTURE ONLY: ctypes wrapper around the plain-C oracle of the int4 MoE layer.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this package.  The
CUDA library never calls it, and nothing here imports the CUDA library.  ``build()`` compiles
``moe_oracle.c`` with gcc (OpenMP, no FMA contraction so each fp32 dequantisation step rounds on
its own).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
               "-shared", "-fPIC", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("H", "I", "E", "k", "group", "has_shared")] + \
        [(n, ctypes.c_void_p) for n in (
            "q_gate", "q_up", "q_down", "s_gate", "b_gate", "s_up", "b_up", "s_down", "b_down",
            "qs_gate", "qs_up", "qs_down", "ss_gate", "bs_gate", "ss_up", "bs_up", "ss_down",
            "bs_down", "router", "router_bias", "shared_gate")]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_dequant.argtypes = [P, P, P, i, i, i, P]
        L.oracle_router_logits.argtypes = [P, P, i, P]
        L.oracle_select.argtypes = [P, i, i, i, P, P]
        L.oracle_shared_gate.argtypes = [P, P, i, P]
        L.oracle_bucket.argtypes = [P, i, i, i, P, P, P]
        L.oracle_expert_ffn.argtypes = [P, i, P, P]
        L.oracle_forward.argtypes = [P, P, i, P, i, P, P, P, P]
        L.oracle_forward_dense.argtypes = [P, P, i, P, i, P]
        L.oracle_set_threads.argtypes = [i]
        L.oracle_max_threads.restype = i
        _lib = L
    return _lib


def _np(t, dtype):
    """torch tensor / numpy array -> C-contiguous numpy array of the given dtype (bit view)."""
    if t is None:
        return None
    if hasattr(t, "detach"):
        import torch
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        a = t.numpy()
    else:
        a = np.ascontiguousarray(t)
    if a.dtype != dtype:
        a = a.view(dtype) if a.dtype.itemsize == np.dtype(dtype).itemsize else a.astype(dtype)
    return np.ascontiguousarray(a)


def _ptr(a):
    return None if a is None else a.ctypes.data


class OracleLayer:
    """Holds host copies of one layer (public layout) and a C view of it."""

    _U32 = ("q_gate", "q_up", "q_down", "qs_gate", "qs_up", "qs_down")
    _U16 = ("s_gate", "b_gate", "s_up", "b_up", "s_down", "b_down",
            "ss_gate", "bs_gate", "ss_up", "bs_up", "ss_down", "bs_down")
    _F32 = ("router", "router_bias", "shared_gate")

    def __init__(self, w: Dict[str, object], H: int, I: int, E: int, k: int, group: int = 64,
                 has_shared: Optional[bool] = None):
        self.arrays = {}
        for n in self._U32:
            self.arrays[n] = _np(w.get(n), np.uint32)
        for n in self._U16:
            self.arrays[n] = _np(w.get(n), np.uint16)
        for n in self._F32:
            self.arrays[n] = _np(w.get(n), np.float32)
        if has_shared is None:
            has_shared = self.arrays["qs_gate"] is not None
        self.H, self.I, self.E, self.k, self.group = H, I, E, k, group
        self.has_shared = bool(has_shared)
        self.c = _Layer(H, I, E, k, group, int(has_shared),
                        *[_ptr(self.arrays[n]) for n in (
                            "q_gate", "q_up", "q_down", "s_gate", "b_gate", "s_up", "b_up",
                            "s_down", "b_down", "qs_gate", "qs_up", "qs_down", "ss_gate",
                            "bs_gate", "ss_up", "bs_up", "ss_down", "bs_down", "router",
                            "router_bias", "shared_gate")])

    @classmethod
    def from_shape(cls, w, shape):
        return cls(w, shape.H, shape.I, shape.E, shape.k, shape.group, shape.has_shared)

    # ---- routing -------------------------------------------------------------------------
    def logits(self, x) -> np.ndarray:
        xb = _np(x, np.uint16)
        T = xb.shape[0]
        out = np.zeros((T, self.E), np.float64)
        lib().oracle_router_logits(ctypes.byref(self.c), _ptr(xb), T, _ptr(out))
        return out

    def route(self, x):
        """-> (idx [T,k] int32, gates [T,k] f64, shared gate [T] f64, logits [T,E] f64)"""
        lg = self.logits(x)
        T = lg.shape[0]
        idx = np.zeros((T, self.k), np.int32)
        g = np.zeros((T, self.k), np.float64)
        lib().oracle_select(_ptr(lg), T, self.E, self.k, _ptr(idx), _ptr(g))
        sg = np.zeros(T, np.float64)
        if self.has_shared:
            xb = _np(x, np.uint16)
            lib().oracle_shared_gate(ctypes.byref(self.c), _ptr(xb), T, _ptr(sg))
        return idx, g, sg, lg

    # ---- forward --------------------------------------------------------------------------
    def forward(self, x, tokens: Optional[Sequence[int]] = None, dense: bool = False):
        """-> y [ntok, H] fp64 for the listed tokens (all tokens when None)."""
        xb = _np(x, np.uint16)
        T = xb.shape[0]
        tk = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, np.int32))
        n = T if tk is None else len(tk)
        y = np.zeros((n, self.H), np.float64)
        if dense:
            lib().oracle_forward_dense(ctypes.byref(self.c), _ptr(xb), T, _ptr(tk), n, _ptr(y))
        else:
            lib().oracle_forward(ctypes.byref(self.c), _ptr(xb), T, _ptr(tk), n, _ptr(y),
                                 None, None, None)
        return y

    def expert_ffn(self, e: int, xt: np.ndarray) -> np.ndarray:
        xt = np.ascontiguousarray(xt, np.float64)
        y = np.zeros(self.H, np.float64)
        lib().oracle_expert_ffn(ctypes.byref(self.c), e, _ptr(xt), _ptr(y))
        return y


def bucket(idx: np.ndarray, E: int):
    """-> (counts [E], offsets [E+1], perm [T*k]) of the stable counting sort by expert."""
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    lib().oracle_bucket(_ptr(idx), T, k, E, _ptr(counts), _ptr(offsets), _ptr(perm))
    return counts, offsets, perm


def dequant(q, s, b, rows: int, cols: int, group: int = 64) -> np.ndarray:
    qa, sa, ba = _np(q, np.uint32), _np(s, np.uint16), _np(b, np.uint16)
    out = np.zeros((rows, cols), np.float32)
    lib().oracle_dequant(_ptr(qa), _ptr(sa), _ptr(ba), rows, cols, group, _ptr(out))
    return out


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())
