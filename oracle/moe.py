"""Routed SwiGLU experts and the weighted combine (oracle, fp64).

The pages describe the MoE layer only as routed experts on top of a dense
backbone (hipfire offload explainer, opening section: attention, state and
LM head run every step, experts only when selected).  The expert FFN and the
combine are the plain SwiGLU reading:
    g = Wg x,  u = Wu x,  h = silu(g) * u = g / (1 + e^-g) * u,
    o = Wd h,  y_t = sum_j w_tj * o_tj   (j = slot order of the router),
with Wg, Wu [I x H] and Wd [H x I] the dequantised HFQ4 matrices (exact
w = zero + scale*q, see hfq4.py).  No shared expert and no biases.

``tc=True`` is the numeric model of the bf16 tensor-core path: weights are
RN_bf16(RN_f32(w)), the activations are already bf16, and everything else
stays fp64.  h is not rounded: the path carries it into the down projection
as two bf16 parts (hi = bf16(h), lo = bf16(h - hi), about 16 significant
bits), whose remaining error is far inside the parity tolerance, whereas a
single bf16 rounding of h would not be a unique result (values near a
rounding boundary go either way with the path's f32 errors).  The pages give
no precision for their tensor-core prefill path (gfx1151 engine README,
"Windows" section), so this is a stated reading.
"""
from __future__ import annotations

import numpy as np

from . import hfq4


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest, ties to even) through f32; returns f64 values."""
    b = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32)).view(np.uint32)
    b = b.astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def expert_hidden(wg: np.ndarray, wu: np.ndarray, x: np.ndarray):
    """(g, u, h) = (Wg x, Wu x, silu(g) * u) for x [H] or [T, H] (rows are
    tokens), fp64."""
    x = np.asarray(x, dtype=np.float64)
    g = x @ wg.T
    u = x @ wu.T
    return g, u, silu(g) * u


def expert_ffn(wg: np.ndarray, wu: np.ndarray, wd: np.ndarray, x: np.ndarray) -> np.ndarray:
    """o = Wd (silu(Wg x) * (Wu x)) for x [H] or [T, H] (rows are tokens)."""
    _, _, h = expert_hidden(wg, wu, x)
    return h @ wd.T


class ExpertCache:
    """Dequantises each packed expert once; experts: uint8 [E, expert_bytes]."""

    def __init__(self, experts: np.ndarray, hidden: int, inter: int, tc: bool = False):
        self.experts, self.hidden, self.inter, self.tc = experts, hidden, inter, tc
        self._w = {}

    def __call__(self, e: int):
        if e not in self._w:
            wg, wu, wd = hfq4.dequantize_expert(self.experts[e], self.hidden, self.inter)
            if self.tc:
                wg, wu, wd = (round_bf16(m.astype(np.float32)) for m in (wg, wu, wd))
            self._w[e] = (wg, wu, wd)
        return self._w[e]


def moe_layer(experts, hidden: int, inter: int, x: np.ndarray, idx: np.ndarray,
              wts: np.ndarray, tc: bool = False) -> np.ndarray:
    """y [T, H] fp64 of the routed layer.

    experts: uint8 [E, expert_bytes] packed layer, or an ExpertCache;
    x: [T, H] activation values; idx int [T, k]; wts [T, k] routing weights."""
    cache = experts if isinstance(experts, ExpertCache) else ExpertCache(experts, hidden, inter, tc)
    x = np.asarray(x, dtype=np.float64)
    T, k = idx.shape
    y = np.zeros((T, hidden), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            wg, wu, wd = cache(int(idx[t, j]))
            y[t] += float(wts[t, j]) * expert_ffn(wg, wu, wd, x[t])
    return y


def moe_dense(experts, hidden: int, inter: int, x: np.ndarray, idx: np.ndarray,
              wts: np.ndarray) -> np.ndarray:
    """Second formulation for cross-checks: y_t = sum over ALL experts e of
    m_te * FFN_e(x_t), with m_te the routing weight if e is selected, else 0."""
    cache = experts if isinstance(experts, ExpertCache) else ExpertCache(experts, hidden, inter)
    x = np.asarray(x, dtype=np.float64)
    T, k = idx.shape
    E = len(cache.experts)
    m = np.zeros((T, E))
    for t in range(T):
        m[t, idx[t]] = wts[t]
    y = np.zeros((T, hidden))
    for e in range(E):
        wg, wu, wd = cache(e)
        y += m[:, e:e + 1] * expert_ffn(wg, wu, wd, x)
    return y


def residual_stack(layer_caches, logits: np.ndarray, x0: np.ndarray, k: int, route_fn,
                   on_layer=None):
    """A decode stack of MoE layers joined by a bf16 residual stream:
    x_{l+1} = RN_bf16(x_l + y_l), with layer l routed on logits[l].

    layer_caches: one ExpertCache per layer; logits f32 [L, T, E]; x0 [T, H]
    bf16 values.  Returns (ys [L, T, H] fp64, xs [L+1, T, H] bf16 values)."""
    L = len(layer_caches)
    xs = [np.asarray(x0, dtype=np.float64)]
    ys = []
    for l in range(L):
        idx, wts = route_fn(logits[l], k)
        c = layer_caches[l]
        y = moe_layer(c, c.hidden, c.inter, xs[-1], idx, wts)
        ys.append(y)
        xs.append(round_bf16(xs[-1] + y))
        if on_layer is not None:
            on_layer(l, idx, wts, y)
    return np.stack(ys), np.stack(xs)
