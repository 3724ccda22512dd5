"""Seeded synthetic inputs for the int4 MoE layer (shared by the oracle-side tests and the CUDA path).

This module draws random numbers and nothing else: it holds none of the layer's arithmetic
(no routing, no dequantisation, no matmul).  Everything it returns is in the library's public
("natural") layout, the one `include/moe.h` documents:

* packed weights ``q_*``: uint32 words, ``[rows, cols/8]``; nibble ``j`` (bits ``4j..4j+3``) of
  word ``w`` is element ``8w+j`` of the row, low nibble first;
* per-group scale/bias ``s_*``/``b_*``: bfloat16 ``[rows, cols/group]``, group = 64 input columns;
* router ``[E, H]`` fp32, optional router bias ``[E]`` fp32, shared-expert gate vector ``[H]`` fp32;
* activations ``x``: bfloat16 ``[T, H]``.

Distributions (the workload definition of the MoE layer this library implements): quant values
uniform over 0..15 (so every packed word is 32 uniform random bits), scales U(0.005, 0.02) rounded
to bf16, biases ``-8 * scale`` (exact in bf16), router and shared-gate weights N(0, 0.02) in fp32,
activations N(0, 1) rounded to bf16.  The skewed workloads add a per-expert router bias
``-s * ln(rank)`` over a random permutation of the experts (a log-Zipf(s) prior).

Streams: every (workload seed, layer) pair has its own torch.Generator for weights, and every
(seed, layer, chunk) its own generator for activations; redraws of activation rows come from the
next draws of that same activation stream.  The CPU and CUDA torch generators give different
streams for the same seed: tests draw on the CPU and copy to the GPU; the benchmark draws its
40-layer stacks directly on the GPU.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Shape:
    """Shapes of one MoE-layer workload."""
    name: str
    T: int            # tokens per forward call (one chunk)
    H: int            # hidden size
    E: int            # routed experts
    k: int            # experts kept per token
    I: int            # expert SwiGLU intermediate size
    group: int = 64   # quantisation group along the input dimension
    has_shared: bool = True
    layers: int = 1   # distinct layers (timing loops cycle through them)
    chunks: int = 1   # forward calls per layer (long prompts are split into chunks)
    zipf_s: Optional[float] = None
    seed: int = 0


# The five workloads: a tiny layer for parity, batch-1 decode over 40 layers, two prefill sizes
# and a 16384-token prefill processed as four 4096-token chunks over 40 layers.
WORKLOADS: Dict[str, Shape] = {
    "tiny": Shape("tiny", T=8, H=256, E=16, k=2, I=128, seed=0),
    "decode": Shape("decode", T=1, H=2048, E=256, k=8, I=512, layers=40, seed=1),
    "prefill512": Shape("prefill512", T=512, H=2048, E=256, k=8, I=512, seed=2),
    "prefill4k_zipf": Shape("prefill4k_zipf", T=4096, H=2048, E=256, k=8, I=512, zipf_s=1.1, seed=3),
    "prefill16k_zipf": Shape("prefill16k_zipf", T=4096, H=2048, E=256, k=8, I=512, layers=40,
                             chunks=4, zipf_s=1.2, seed=4),
}
WORKLOAD_ORDER = ["tiny", "decode", "prefill512", "prefill4k_zipf", "prefill16k_zipf"]


def _gen(device, *key: int) -> torch.Generator:
    # one independent stream per key tuple (plain mixing of small integers into a 63-bit seed)
    s = 0x9E3779B97F4A7C15
    for v in key:
        s = (s * 6364136223846793005 + (v & 0xFFFFFFFF) + 1442695040888963407) % (1 << 63)
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def _words(g: torch.Generator, shape, device) -> torch.Tensor:
    """Uniform 32-bit words, i.e. 8 independent uniform nibbles each (returned as int32)."""
    n = 1
    for d in shape:
        n *= d
    b = torch.randint(0, 256, (n * 4,), dtype=torch.uint8, generator=g, device=device)
    return b.view(torch.int32).view(*shape)


def _scales(g: torch.Generator, shape, device):
    u = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    s = (0.005 + 0.015 * u).to(torch.bfloat16)
    b = (s.float() * -8.0).to(torch.bfloat16)   # exact: a power-of-two multiple of a bf16
    return s, b


def _matrix(g, n_mats, rows, cols, group, device):
    q = _words(g, (n_mats, rows, cols // 8), device) if n_mats else _words(g, (rows, cols // 8), device)
    shp = (n_mats, rows, cols // group) if n_mats else (rows, cols // group)
    s, b = _scales(g, shp, device)
    return q, s, b


def make_layer(shape: Shape, layer: int = 0, device="cpu") -> Dict[str, Optional[torch.Tensor]]:
    """All weights of one layer, drawn in a fixed order from the (seed, layer) stream."""
    g = _gen(device, shape.seed, layer, 0x57)
    H, I, E, G = shape.H, shape.I, shape.E, shape.group
    w: Dict[str, Optional[torch.Tensor]] = {}
    w["q_gate"], w["s_gate"], w["b_gate"] = _matrix(g, E, I, H, G, device)
    w["q_up"], w["s_up"], w["b_up"] = _matrix(g, E, I, H, G, device)
    w["q_down"], w["s_down"], w["b_down"] = _matrix(g, E, H, I, G, device)
    if shape.has_shared:
        w["qs_gate"], w["ss_gate"], w["bs_gate"] = _matrix(g, 0, I, H, G, device)
        w["qs_up"], w["ss_up"], w["bs_up"] = _matrix(g, 0, I, H, G, device)
        w["qs_down"], w["ss_down"], w["bs_down"] = _matrix(g, 0, H, I, G, device)
        w["shared_gate"] = torch.randn(H, generator=g, device=device, dtype=torch.float32) * 0.02
    else:
        for n in ("qs_gate", "ss_gate", "bs_gate", "qs_up", "ss_up", "bs_up",
                  "qs_down", "ss_down", "bs_down", "shared_gate"):
            w[n] = None
    w["router"] = torch.randn(E, H, generator=g, device=device, dtype=torch.float32) * 0.02
    w["router_bias"] = zipf_bias(shape.E, shape.zipf_s, g, device) if shape.zipf_s else None
    return w


def zipf_bias(E: int, s: float, g: torch.Generator, device="cpu") -> torch.Tensor:
    """Per-expert log-Zipf(s) prior: expert perm[r-1] gets -s*ln(r), rank r = 1..E."""
    perm = torch.randperm(E, generator=g, device=device)
    ranks = torch.empty(E, dtype=torch.float64, device=device)
    ranks[perm] = torch.arange(1, E + 1, dtype=torch.float64, device=device)
    return (-s * torch.log(ranks)).to(torch.float32)


class ActivationStream:
    """Activation rows for one (seed, layer, chunk): N(0,1) rounded to bf16, drawn in order."""

    def __init__(self, shape: Shape, layer: int = 0, chunk: int = 0, device="cpu"):
        self.H = shape.H
        self.device = device
        self.g = _gen(device, shape.seed, layer, chunk, 0xA7)

    def draw(self, n: int) -> torch.Tensor:
        return torch.randn(n, self.H, generator=self.g, device=self.device,
                           dtype=torch.float32).to(torch.bfloat16)


def make_x(shape: Shape, layer: int = 0, chunk: int = 0, device="cpu", T: Optional[int] = None):
    return ActivationStream(shape, layer, chunk, device).draw(shape.T if T is None else T)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its bit patterns (no arithmetic)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")


def layer_bytes(shape: Shape) -> int:
    """Bytes of one layer's weights in the public layout (packed nibbles + bf16 scale/bias + fp32)."""
    n_exp = shape.E + (1 if shape.has_shared else 0)
    per = 3 * shape.I * shape.H // 2 + 3 * shape.I * shape.H // shape.group * 4
    extra = shape.E * shape.H * 4 + (shape.H * 4 if shape.has_shared else 0) + \
        (shape.E * 4 if shape.zipf_s else 0)
    return n_exp * per + extra


def shape_with(shape: Shape, **kw) -> Shape:
    return dataclasses.replace(shape, **kw)


__all__ = ["Shape", "WORKLOADS", "WORKLOAD_ORDER", "make_layer", "make_x", "ActivationStream",
           "zipf_bias", "bf16_bits", "layer_bytes", "shape_with"]

