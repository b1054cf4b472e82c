"""Pins for the oracle's expert FFN and combine (no GPU).

* one expert, top-1: the layer is a textbook SwiGLU MLP, written out here
  with plain loops over the dequantised weights;
* constant weights and inputs: a closed form;
* the sparse combine agrees with the dense formulation over all experts;
* the bf16 (tensor-core) model equals the exact one when every rounded value
  is already representable;
* planted mistakes (dropped weight, wrong activation, transposed down
  projection) are caught.
"""
import math

import numpy as np
import pytest

from oracle import hfq4, moe, route


def _pack_layer(E, H, I, seed):
    rng = np.random.default_rng(seed)
    ex = []
    for _ in range(E):
        g = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
        u = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
        d = (rng.standard_normal((H, I)) * 0.02).astype(np.float32)
        ex.append(hfq4.pack_expert(g, u, d))
    return np.stack(ex)


def test_silu_values():
    assert moe.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(moe.silu(np.array([1.0])), [1 / (1 + math.exp(-1))], rtol=1e-15)
    np.testing.assert_allclose(moe.silu(np.array([40.0])), [40.0], rtol=1e-15)


def test_single_expert_top1_is_textbook_swiglu():
    H, I = 256, 128
    ex = _pack_layer(1, H, I, 11)
    wg, wu, wd = hfq4.dequantize_expert(ex[0], H, I)
    x = np.random.default_rng(12).standard_normal((2, H))
    idx = np.zeros((2, 1), dtype=np.int32)
    w = np.ones((2, 1))
    y = moe.moe_layer(ex, H, I, x, idx, w)
    for t in range(2):
        h = []
        for i in range(I):
            g = sum(wg[i, c] * x[t, c] for c in range(H))
            u = sum(wu[i, c] * x[t, c] for c in range(H))
            h.append(g / (1.0 + math.exp(-g)) * u)
        for r in range(0, H, 17):
            ref = sum(wd[r, i] * h[i] for i in range(I))
            assert abs(y[t, r] - ref) <= 1e-12 * (1 + abs(ref))


def test_constant_weights_closed_form():
    # every block: scale s, zero z, all q = c  =>  every weight is w = z + s*c
    H, I = 512, 256
    s, z, c = 0.0625, -0.25, 9                       # w = 0.3125
    w = z + s * c
    def mat(R, C):
        nb = hfq4.blocks_per_row(C)
        return hfq4.pack_blocks(np.full((R, nb), s, np.float32), np.full((R, nb), z, np.float32),
                                np.full((R, nb * 256), c, np.uint8))
    ex = np.concatenate([mat(I, H), mat(I, H), mat(H, I)])[None, :]
    a = 0.01
    x = np.full((1, H), a)
    y = moe.moe_layer(np.repeat(ex, 3, axis=0), H, I, x, np.array([[2, 0, 1]], np.int32),
                      np.array([[0.5, 0.3, 0.2]]))
    g = w * H * a
    h = g / (1 + math.exp(-g)) * g
    o = w * I * h
    np.testing.assert_allclose(y, np.full((1, H), o), rtol=1e-13)


def test_sparse_equals_dense():
    E, H, I = 6, 256, 128
    ex = _pack_layer(E, H, I, 21)
    rng = np.random.default_rng(22)
    x = rng.standard_normal((4, H))
    idx, wts = route.route(rng.standard_normal((4, E)).astype(np.float32), 3)
    cache = moe.ExpertCache(ex, H, I)
    ys = moe.moe_layer(cache, H, I, x, idx, wts)
    yd = moe.moe_dense(cache, H, I, x, idx, wts)
    np.testing.assert_allclose(ys, yd, rtol=1e-12, atol=1e-14)


def test_tc_model_equals_exact_on_representable_values():
    # weights z + s*q with few significant bits, x and h forced to bf16 values:
    # the bf16 model must then be identical to the exact one
    H, I = 256, 128
    def mat(R, C, seed):
        nb = hfq4.blocks_per_row(C)
        q = np.random.default_rng(seed).integers(0, 16, (R, nb * 256)).astype(np.uint8)
        return hfq4.pack_blocks(np.full((R, nb), 0.125, np.float32),
                                np.full((R, nb), -1.0, np.float32), q)
    ex = np.concatenate([mat(I, H, 1), mat(I, H, 2), mat(H, I, 3)])[None, :]
    x = np.round(np.random.default_rng(4).standard_normal((1, H)) * 4) / 4
    c_exact, c_tc = moe.ExpertCache(ex, H, I), moe.ExpertCache(ex, H, I, tc=True)
    for e in (0,):
        for m0, m1 in zip(c_exact(e), c_tc(e)):
            np.testing.assert_array_equal(m0, m1)
    one = (np.zeros((1, 1), np.int32), np.ones((1, 1)))
    y0 = moe.moe_layer(c_exact, H, I, x, *one)
    y1 = moe.moe_layer(c_tc, H, I, x, *one)
    wg, wu, wd = c_exact(0)
    g, u = wg @ x[0], wu @ x[0]
    h = moe.silu(g) * u
    assert np.array_equal(y1[0], h @ wd.T)           # h is not rounded in the model
    assert np.array_equal(y0, y1)


def test_round_bf16():
    v = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.0 ** -130, 3.0e38])
    r = moe.round_bf16(v)
    assert r[0] == 1.0
    assert r[1] == 1.0                     # tie -> even
    assert r[2] == 1.0 + 2 * 2**-7         # tie -> even (up)
    assert r[4] == 2.9999999521443642e38 or np.isfinite(r[4])


def test_residual_stack_composes_layers():
    E, H, I = 4, 256, 128
    caches = [moe.ExpertCache(_pack_layer(E, H, I, 30 + l), H, I) for l in range(2)]
    rng = np.random.default_rng(33)
    x0 = moe.round_bf16(rng.standard_normal((1, H)))
    logits = rng.standard_normal((2, 1, E)).astype(np.float32)
    ys, xs = moe.residual_stack(caches, logits, x0, 2, route.route)
    i0, w0 = route.route(logits[0], 2)
    y0 = moe.moe_layer(caches[0], H, I, x0, i0, w0)
    x1 = moe.round_bf16(x0 + y0)
    i1, w1 = route.route(logits[1], 2)
    np.testing.assert_array_equal(ys[0], y0)
    np.testing.assert_array_equal(xs[1], x1)
    np.testing.assert_array_equal(ys[1], moe.moe_layer(caches[1], H, I, x1, i1, w1))


# --- planted mistakes ----------------------------------------------------------

def _reference_small():
    E, H, I = 3, 256, 128
    ex = _pack_layer(E, H, I, 41)
    x = np.random.default_rng(42).standard_normal((2, H))
    idx, wts = route.route(np.random.default_rng(43).standard_normal((2, E)).astype(np.float32), 2)
    return ex, H, I, x, idx, wts


def test_planted_dropped_combine_weight_is_caught():
    ex, H, I, x, idx, wts = _reference_small()
    good = moe.moe_dense(ex, H, I, x, idx, wts)
    bad = moe.moe_layer(ex, H, I, x, idx, np.ones_like(wts))
    assert not np.allclose(good, bad, rtol=1e-6)


def test_planted_wrong_activation_is_caught(monkeypatch):
    ex, H, I, x, idx, wts = _reference_small()
    cache = moe.ExpertCache(ex, H, I)
    wg, wu, wd = cache(0)
    g, u = wg @ x[0], wu @ x[0]
    ref = sum(wd[5, i] * (g[i] / (1 + math.exp(-g[i]))) * u[i] for i in range(I))
    monkeypatch.setattr(moe, "silu", lambda v: v / (1.0 + np.exp(v)))      # sign slip
    got = moe.expert_ffn(wg, wu, wd, x[0])[5]
    assert abs(got - ref) > 1e-9


def test_planted_transposed_down_is_caught():
    E, H, I = 1, 256, 256
    ex = _pack_layer(E, H, I, 51)
    wg, wu, wd = hfq4.dequantize_expert(ex[0], H, I)
    x = np.random.default_rng(52).standard_normal(H)
    a = moe.expert_ffn(wg, wu, wd, x)
    b = moe.expert_ffn(wg, wu, wd.T.copy(), x)
    assert not np.allclose(a, b, rtol=1e-6)


def test_grouped_oracle_equals_moe_layer():
    """The expert-by-expert oracle the full-size GPU checks use
    (tests/gpu_util.py oracle_rows) gives moe_layer's y, in the exact and the
    bf16 tensor-core model, for any subset of tokens."""
    import synth
    from synth import workloads as W
    from tests.gpu_util import OraclePackedLayer, oracle_rows

    w = W.WORKLOADS[1]
    T, k = 8, w.top_k
    x, _ = W.activations(w, 0, T)
    x_bits = synth.to_bf16_bits(x.astype(np.float32))
    xv = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    idx, wts = route.route(W.logits(w, 0, 0, T), k)
    rows = np.array([1, 4, 6])
    for tc in (False, True):
        cache = moe.ExpertCache(OraclePackedLayer(w, 0), w.hidden, w.inter, tc=tc)
        ref = moe.moe_layer(cache, w.hidden, w.inter, xv, idx, wts)
        y = oracle_rows(w, 0, x_bits, idx, wts, rows, tc=tc, workers=0)
        np.testing.assert_allclose(y, ref[rows], rtol=1e-12, atol=1e-15)
