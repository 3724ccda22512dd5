"""Test-side helpers: seeded layers, and activations with a guaranteed top-(k+1) logit gap.

The gap rule: every token's k+1 largest fp64 router logits (bias included) are at least
``min_gap`` apart pairwise-adjacent, so both the selected set and its order are stable under
fp32 rounding on the GPU.  Rows that miss it are redrawn from the next draws of the same seeded
activation stream.  The logits come from the oracle, so this helper lives with the tests.
"""
import numpy as np

import oracle
from bit_grouped_expert_router_b200 import synth


def min_adjacent_gap(logits: np.ndarray, k: int) -> np.ndarray:
    m = min(k + 1, logits.shape[1])
    top = -np.sort(-logits, axis=1)[:, :m]
    if m < 2:
        return np.full(logits.shape[0], np.inf)
    return (top[:, :-1] - top[:, 1:]).min(axis=1)


def gapped_x(shape, ol, layer=0, chunk=0, T=None, min_gap=1e-3, max_rounds=200):
    stream = synth.ActivationStream(shape, layer, chunk)
    x = stream.draw(shape.T if T is None else T)
    for _ in range(max_rounds):
        gaps = min_adjacent_gap(ol.logits(x), shape.k)
        bad = np.nonzero(gaps < min_gap)[0]
        if len(bad) == 0:
            return x
        x[bad] = stream.draw(len(bad))
    raise RuntimeError("could not draw activations meeting the logit gap")


def layer_and_x(name_or_shape, layer=0, chunk=0, T=None):
    shape = synth.WORKLOADS[name_or_shape] if isinstance(name_or_shape, str) else name_or_shape
    w = synth.make_layer(shape, layer)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol, layer, chunk, T)
    return shape, w, ol, x
