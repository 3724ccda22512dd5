"""Pins for the CPU oracle, against things other than itself (CPU only).

* dequantisation: hand-worked words (tests/golden/dequant_nibbles.txt) and the all-zero code;
* routing: numpy fp64 matmul for the logits, numpy's stable sort for the selection (ties go to
  the lower expert index), scipy's softmax for the renormalised gates, scipy's expit for the
  shared gate; invariants (gates sum to 1, k distinct experts); k = E reduces to a full softmax;
  a +100 bias on 8 experts routes every token to them;
* bucketing: numpy bincount and numpy's stable argsort; permute-then-unpermute is the identity;
* expert FFN and combine: closed forms with constant per-expert weights, a single dense SwiGLU
  MLP (E = 1, k = 1, no shared expert) against numpy matmuls, the shared expert alone, and the
  sparse oracle against dense evaluation of all E experts with the unselected gates zeroed.
"""
import os

import numpy as np
import pytest
import torch
from scipy.special import expit, softmax

import oracle
from bit_grouped_expert_router_b200 import synth
from helpers import gapped_x, min_adjacent_gap

HERE = os.path.dirname(os.path.abspath(__file__))
TINY = synth.WORKLOADS["tiny"]
MEDIUM = synth.Shape("medium", T=24, H=512, E=32, k=4, I=128, zipf_s=1.1, seed=11)


def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _xf64(x):
    return x.float().double().numpy()


# --------------------------------------------------------------------------------------------
# dequantisation
def test_dequant_hand_worked_words():
    rows = []
    with open(os.path.join(HERE, "golden", "dequant_nibbles.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            p = line.split()
            rows.append((int(p[0], 16), int(p[1], 16), int(p[2], 16), [float(v) for v in p[3:]]))
    assert len(rows) >= 4
    for word, s, b, want in rows:
        q = np.array([[word]], np.uint32)
        sa = np.array([[s]], np.uint16)
        ba = np.array([[b]], np.uint16)
        got = oracle.dequant(q, sa, ba, rows=1, cols=8, group=8)
        assert got.tolist() == [want], (hex(word), got, want)


def test_dequant_groups_and_rows():
    # two rows x 128 columns, two groups per row with distinct scales: row r, group c gets
    # scale 2^-(r+c) and bias -(8+c); every word is 0x76543210 (elements 0..7 repeating)
    q = np.full((2, 16), 0x76543210, np.uint32)
    s = np.array([[2.0 ** -(r + c) for c in range(2)] for r in range(2)], np.float32)
    b = np.array([[-(8.0 + c) for c in range(2)] for r in range(2)], np.float32)
    W = oracle.dequant(q, _bf16_bits(s).reshape(2, 2), _bf16_bits(b).reshape(2, 2), 2, 128, 64)
    for r in range(2):
        for col in range(128):
            c = col // 64
            assert W[r, col] == (col % 8) * 2.0 ** -(r + c) - (8.0 + c)


def test_dequant_all_eights_is_zero():
    shape = TINY
    w = synth.make_layer(shape)
    q = np.full((shape.I, shape.H // 8), 0x88888888, np.uint32)
    s = w["s_gate"][0]
    W = oracle.dequant(q, s, (s.float() * -8).to(torch.bfloat16), shape.I, shape.H)
    assert (W == 0).all()


# --------------------------------------------------------------------------------------------
# routing
@pytest.mark.parametrize("shape", [TINY, MEDIUM], ids=["tiny", "medium"])
def test_route_against_numpy_sort_and_softmax(shape):
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    idx, g, sg, lg = ol.route(x)
    X = _xf64(x)
    ref_l = X @ w["router"].double().numpy().T
    if w["router_bias"] is not None:
        ref_l = ref_l + w["router_bias"].double().numpy()[None, :]
    np.testing.assert_allclose(lg, ref_l, rtol=0, atol=1e-12)
    order = np.argsort(-ref_l, axis=1, kind="stable")[:, : shape.k]
    assert (idx == order).all()
    p = softmax(ref_l, axis=1)
    sel = np.take_along_axis(p, order, axis=1)
    np.testing.assert_allclose(g, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(sg, expit(X @ w["shared_gate"].double().numpy()), rtol=1e-12)
    # invariants
    assert np.abs(g.sum(axis=1) - 1).max() <= 1e-12
    assert all(len(set(r)) == shape.k for r in idx.tolist())
    assert (np.diff(np.take_along_axis(lg, idx, 1), axis=1) < 0).all()
    assert (min_adjacent_gap(lg, shape.k) >= 1e-3).all()


def test_route_ties_go_to_lower_index():
    shape = synth.shape_with(TINY, T=4)
    w = synth.make_layer(shape)
    R = w["router"].clone()
    R[9] = R[3] * 50          # experts 3 and 9 identical and dominant
    R[3] = R[9]
    w["router"] = R
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = torch.ones(4, shape.H, dtype=torch.bfloat16) * torch.sign(R[3]).to(torch.bfloat16)
    idx, g, _, lg = ol.route(x)
    assert (lg[:, 3] == lg[:, 9]).all()
    assert idx[:, 0].tolist() == [3] * 4 and idx[:, 1].tolist() == [9] * 4
    np.testing.assert_allclose(g, 0.5, rtol=1e-15)


def test_route_k_equals_E_is_full_softmax():
    shape = synth.Shape("kE", T=6, H=128, E=8, k=8, I=64, seed=5)
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = synth.make_x(shape)
    idx, g, _, lg = ol.route(x)
    full = softmax(lg, axis=1)
    np.testing.assert_allclose(g, np.take_along_axis(full, idx, 1), rtol=1e-12)
    assert (np.sort(idx, axis=1) == np.arange(8)[None, :]).all()


def test_route_large_bias_forces_the_chosen_experts():
    shape = synth.Shape("forced", T=16, H=256, E=32, k=8, I=64, seed=6)
    w = synth.make_layer(shape)
    chosen = [1, 4, 7, 10, 17, 22, 28, 31]
    bias = torch.zeros(shape.E)
    bias[chosen] = 100.0
    w["router_bias"] = bias
    ol = oracle.OracleLayer.from_shape(w, shape)
    idx, _, _, _ = ol.route(synth.make_x(shape))
    assert all(sorted(r) == chosen for r in idx.tolist())
    counts, offsets, _ = oracle.bucket(idx, shape.E)
    assert counts[chosen].tolist() == [shape.T] * 8 and counts.sum() == shape.T * 8


# --------------------------------------------------------------------------------------------
# bucketing
@pytest.mark.parametrize("T,E,k", [(0, 16, 2), (1, 16, 2), (7, 16, 4), (64, 256, 8), (300, 40, 8)])
def test_bucket_against_numpy(T, E, k):
    rng = np.random.default_rng(T * 131 + E)
    idx = np.array([rng.choice(E, k, replace=False) for _ in range(T)], np.int32).reshape(T, k)
    counts, offsets, perm = oracle.bucket(idx, E)
    flat = idx.ravel()
    assert (counts == np.bincount(flat, minlength=E)).all()
    assert offsets[0] == 0 and offsets[-1] == T * k and (np.diff(offsets) == counts).all()
    assert (perm == np.argsort(flat, kind="stable")).all()
    v = rng.standard_normal(T * k)
    back = np.empty_like(v)
    back[perm] = v[perm]
    assert (back == v).all()
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg // k) > 0).all()


# --------------------------------------------------------------------------------------------
# expert FFN and combine
def _const_layer(shape, codes):
    """Layer whose every matrix of expert e is constant: W = (q_e - 8) * s with s = 1 (gate, up)
    or W = q_e * 0.5 - 4 (down).  codes(e) -> (q_gate, q_up, q_down)."""
    w = synth.make_layer(shape)
    n = shape.E + 1

    def fill(nib, rows, cols, scale, bias, e_count):
        word = int("".join([format(nib, "x")] * 8), 16)
        q = torch.full((e_count, rows, cols // 8), word, dtype=torch.int64).to(torch.int32) \
            if word < 2 ** 31 else torch.full((e_count, rows, cols // 8), word - 2 ** 32, dtype=torch.int32)
        s = torch.full((e_count, rows, cols // 64), scale).to(torch.bfloat16)
        b = torch.full((e_count, rows, cols // 64), bias).to(torch.bfloat16)
        return q, s, b

    for name, (rows, cols, scale, bias, col) in {
        "gate": (shape.I, shape.H, 1.0, -8.0, 0),
        "up": (shape.I, shape.H, 1.0, -8.0, 1),
        "down": (shape.H, shape.I, 0.5, -4.0, 2),
    }.items():
        qs, ss, bs = [], [], []
        for e in range(n):
            q, s, b = fill(codes(e)[col], rows, cols, scale, bias, 1)
            qs.append(q); ss.append(s); bs.append(b)
        w["q_" + name] = torch.cat(qs[:-1]); w["s_" + name] = torch.cat(ss[:-1]); w["b_" + name] = torch.cat(bs[:-1])
        w["qs_" + name] = qs[-1][0]; w["ss_" + name] = ss[-1][0]; w["bs_" + name] = bs[-1][0]
    return w


def test_forward_closed_form_constant_experts():
    shape = synth.Shape("const", T=12, H=256, E=16, k=3, I=128, seed=7)
    codes = lambda e: (9 + e % 4, 10 + e % 5, 10 + e % 3)
    w = _const_layer(shape, codes)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = (synth.make_x(shape).float() * 0.05).to(torch.bfloat16)
    y = ol.forward(x)
    X = _xf64(x)
    S = X.sum(axis=1)
    lg = X @ w["router"].double().numpy().T
    order = np.argsort(-lg, axis=1, kind="stable")[:, : shape.k]
    p = np.take_along_axis(softmax(lg, axis=1), order, 1)
    g = p / p.sum(axis=1, keepdims=True)
    sg = expit(X @ w["shared_gate"].double().numpy())

    def expert_out(e, s):
        a, u, d = codes(e)[0] - 8, codes(e)[1] - 8, codes(e)[2] * 0.5 - 4
        gz = a * s
        return d * shape.I * (gz / (1 + np.exp(-gz))) * (u * s)

    ref = np.zeros(shape.T)
    for t in range(shape.T):
        ref[t] = sum(g[t, j] * expert_out(order[t, j], S[t]) for j in range(shape.k))
        ref[t] += sg[t] * expert_out(shape.E, S[t])
    np.testing.assert_allclose(y, np.repeat(ref[:, None], shape.H, axis=1), rtol=1e-12, atol=1e-12)


def test_forward_zero_weights_give_zero():
    # code 8 with (s, b) = (1, -8) for gate/up and (0.5, -4) for down: every weight is zero
    shape = synth.shape_with(TINY, T=5)
    w = _const_layer(shape, lambda e: (8, 8, 8))
    ol = oracle.OracleLayer.from_shape(w, shape)
    assert (ol.forward(synth.make_x(shape)) == 0).all()


def _dequant_all(w, shape, prefix, e=None):
    names = {"gate": (shape.I, shape.H), "up": (shape.I, shape.H), "down": (shape.H, shape.I)}
    out = {}
    for n, (r, c) in names.items():
        q, s, b = w["q" + prefix + "_" + n], w["s" + prefix + "_" + n], w["b" + prefix + "_" + n]
        if e is not None:
            q, s, b = q[e], s[e], b[e]
        out[n] = oracle.dequant(q, s, b, r, c).astype(np.float64)
    return out


def _swiglu(W, X):
    gz = X @ W["gate"].T
    return ((gz * expit(gz)) * (X @ W["up"].T)) @ W["down"].T


def test_single_expert_is_a_dense_swiglu_mlp():
    shape = synth.Shape("mlp", T=6, H=256, E=1, k=1, I=192, has_shared=False, seed=8)
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = synth.make_x(shape)
    np.testing.assert_allclose(ol.forward(x), _swiglu(_dequant_all(w, shape, "", 0), _xf64(x)),
                               rtol=1e-11, atol=1e-11)


def test_shared_expert_alone():
    shape = synth.Shape("shared", T=5, H=256, E=4, k=2, I=128, seed=9)
    w = synth.make_layer(shape)
    zero_word = torch.tensor(0x88888888 - 2 ** 32, dtype=torch.int32)
    for n in ("gate", "up", "down"):
        w["q_" + n] = torch.full_like(w["q_" + n], int(zero_word))
        w["b_" + n] = (w["s_" + n].float() * -8).to(torch.bfloat16)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = synth.make_x(shape)
    X = _xf64(x)
    sg = expit(X @ w["shared_gate"].double().numpy())
    ref = sg[:, None] * _swiglu(_dequant_all(w, shape, "s"), X)
    np.testing.assert_allclose(ol.forward(x), ref, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("shape", [TINY, synth.shape_with(MEDIUM, T=6)], ids=["tiny", "medium"])
def test_sparse_equals_dense_with_zeroed_gates(shape):
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    ys = ol.forward(x)
    yd = ol.forward(x, dense=True)
    assert np.linalg.norm(ys - yd) <= 1e-12 * np.linalg.norm(yd)


def test_sparse_equals_dense_at_the_full_layer_shapes():
    """The same check at the full layer shapes (H = 2048, E = 256, k = 8, I = 512, shared
    expert): a few tokens through all 256 experts with the unselected gates zeroed."""
    shape = synth.Shape("full_dense", T=3, H=2048, E=256, k=8, I=512, seed=1)
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    ys = ol.forward(x)
    yd = ol.forward(x, dense=True)
    assert np.linalg.norm(ys - yd) <= 1e-12 * np.linalg.norm(yd)


def test_token_subset_matches_full_run():
    shape = TINY
    w = synth.make_layer(shape)
    ol = oracle.OracleLayer.from_shape(w, shape)
    x = gapped_x(shape, ol)
    full = ol.forward(x)
    sub = ol.forward(x, tokens=[5, 0, 7])
    assert (sub == full[[5, 0, 7]]).all()
