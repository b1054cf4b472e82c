"""Workload recipes: the five synthetic configurations of the MoE layer.

Every tensor is a pure function of (seed, coordinates) through the Philox
generator in this package, so the oracle and the GPU path receive identical
inputs.  Nothing here computes a step of the MoE method; routing statistics
that the recipes need (the skew calibration of the verify workload and the
selection counts used for hot placement) use numpy's partition as a plain
library primitive on the synthetic logits.

Shapes follow the pages: the hipfire offload explainer's sample model (40
layers with 408 MiB of HFQ4 experts each, "placement" section), the
512-expert, 48-layer model of the Strata report ("model and engine" section),
top-8 routing (explainer, first section), MTP-style verify batches and
prefill chunks.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np

from . import (STREAM_ACT, STREAM_LOGIT, STREAM_ROUTER, bf16_bits_to_f32, normal, normal_fine,
               to_bf16_bits, uniform, weights)

SEED_BASE = 0x48465134
WEIGHT_SIGMA = 0.02
ROUTER_SIGMA = 0.02
CALIB_TOKEN0 = 1 << 24   # token ids >= this are calibration tokens, disjoint from workload tokens


def seed_of(config_id: int) -> int:
    return SEED_BASE + config_id


@dataclass(frozen=True)
class Workload:
    config_id: int
    name: str
    layers: int
    hidden: int
    inter: int
    experts: int
    top_k: int
    tokens: tuple          # token counts the workload is run at
    act_dtype: str         # "f32" or "bf16"
    logits: str            # "normal" | "skewed" | "zipf"
    n_hot: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return seed_of(self.config_id)


WORKLOADS = {
    1: Workload(1, "tiny moe layer h256 i128 e16 top4 t8", 1, 256, 128, 16, 4, (8,), "f32", "normal"),
    2: Workload(2, "decode stack l40 h2048 i512 e256 top8 t1", 40, 2048, 512, 256, 8, (1,), "bf16",
                "normal"),
    3: Workload(3, "verify stack l48 h2048 i512 e512 top8 t1/2/5/8 skewed", 48, 2048, 512, 512, 8,
                (1, 2, 5, 8), "bf16", "skewed", n_hot=51),
    4: Workload(4, "prefill chunk l1 h2048 i512 e512 top8 t512/2048/8192 zipf1.1", 1, 2048, 512, 512,
                8, (512, 2048, 8192), "bf16", "zipf", extra={"zipf_s": 1.1}),
    5: Workload(5, "offload sweep l48 h2048 i512 e512 top8 t1 host layers N..47", 48, 2048, 512, 512,
                8, (1,), "bf16", "skewed", n_hot=51,
                extra={"resident_layers": (48, 36, 24, 13, 0), "hot_per_layer": (0, 51)}),
}


# ------------------------------------------------------------- activations

def activations_f32(w: Workload, token0: int, T: int) -> np.ndarray:
    """x ~ N(0,1) as f32 [T, H] (token ids token0..token0+T-1)."""
    return normal(w.seed, STREAM_ACT, 0, token0, T, w.hidden, 1.0)


def activations(w: Workload, token0: int, T: int):
    """Activations in the workload's dtype: (array, dtype_name).

    f32 workloads return f32; bf16 workloads return uint16 bf16 bit patterns
    (round to nearest even of the f32 sample)."""
    x = activations_f32(w, token0, T)
    if w.act_dtype == "bf16":
        return to_bf16_bits(x), "bf16"
    return x, "f32"


def activations_value(w: Workload, token0: int, T: int) -> np.ndarray:
    """The activations' exact values as f64 [T, H]."""
    x, dt = activations(w, token0, T)
    return (bf16_bits_to_f32(x) if dt == "bf16" else x).astype(np.float64)


# ------------------------------------------------------------------ logits

def router_weights(w: Workload, layer: int = 0) -> np.ndarray:
    """Router matrix Wr ~ N(0, 0.02) f32 [E, H]."""
    return normal(w.seed, STREAM_ROUTER, layer, 0, w.experts, w.hidden, ROUTER_SIGMA)


def logits(w: Workload, layer: int, token0: int, T: int) -> np.ndarray:
    """Router logits f32 [T, E] for tokens token0.. at one layer."""
    if w.logits == "normal":
        out = normal_fine(w.seed, STREAM_LOGIT, layer, token0, T, w.experts, 1.0)
    elif w.logits == "skewed":
        beta = skew_beta(w)
        out = normal_fine(w.seed, STREAM_LOGIT, layer, token0, T, w.experts, 1.0)
        out[:, hot_set(w, layer)] += np.float32(beta)
    elif w.logits == "zipf":
        out = zipf_logits(w, layer, token0, T)
    else:
        raise ValueError(w.logits)
    # exact ties are rare; both sides break them towards the lower expert index
    return out


def logits_stack(w: Workload, token0: int, T: int) -> np.ndarray:
    """Logits for every layer: f32 [L, T, E]."""
    return np.stack([logits(w, l, token0, T) for l in range(w.layers)])


def hot_set(w: Workload, layer: int) -> np.ndarray:
    """The seeded set of n_hot experts that the skewed router favours."""
    rng = np.random.default_rng([w.seed, layer, 0x484F54])
    return np.sort(rng.permutation(w.experts)[: w.n_hot])


def _hot_share(noise: np.ndarray, hot: np.ndarray, beta: float, k: int) -> float:
    l = noise.copy()
    l[:, hot] += np.float32(beta)
    top = np.argpartition(-l, k - 1, axis=1)[:, :k]
    return float(np.isin(top, hot).mean())


def skew_beta(w: Workload, target: float = 0.60, calib_tokens: int = 4096) -> float:
    """Bias that makes the hot set take `target` of the top-k selections.

    Found by bisection on calibration tokens of layer 0 (token ids from
    CALIB_TOKEN0), rounded to f32."""
    return _skew_beta(w.config_id, target, calib_tokens)


@lru_cache(maxsize=None)
def _skew_beta(config_id: int, target: float, calib_tokens: int) -> float:
    w = WORKLOADS[config_id]
    noise = normal_fine(w.seed, STREAM_LOGIT, 0, CALIB_TOKEN0, calib_tokens, w.experts, 1.0)
    hot = hot_set(w, 0)
    lo, hi = 0.0, 8.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if _hot_share(noise, hot, mid, w.top_k) < target:
            lo = mid
        else:
            hi = mid
    return float(np.float32(0.5 * (lo + hi)))


def zipf_popularity(w: Workload, layer: int = 0) -> np.ndarray:
    """Zipf(s) probabilities over a seeded permutation of the experts: p[e]."""
    s = w.extra.get("zipf_s", 1.1)
    ranks = np.arange(1, w.experts + 1, dtype=np.float64)
    p_rank = ranks ** (-s)
    p_rank /= p_rank.sum()
    perm = np.random.default_rng([w.seed, layer, 0x5A4950]).permutation(w.experts)
    p = np.empty(w.experts)
    p[perm] = p_rank
    return p


def zipf_logits(w: Workload, layer: int, token0: int, T: int) -> np.ndarray:
    """log p_e + Gumbel(0,1) noise, f32 [T, E]; Gumbel = -log(-log u)."""
    p = zipf_popularity(w, layer)
    out = np.empty((T, w.experts), dtype=np.float32)
    for t in range(T):
        u = uniform(w.seed, STREAM_LOGIT, layer, token0 + t, w.experts)
        out[t] = (np.log(p) - np.log(-np.log(u))).astype(np.float32)
    return out


def calibration_counts(w: Workload, calib_tokens: int = 1024) -> np.ndarray:
    """Selections per (layer, expert) over calibration tokens: uint32 [L, E].

    Stands in for the pages' decode-heat ranking of experts (the hipfire
    offload explainer's expert-hotset sidecar, "placement" section)."""
    counts = np.zeros((w.layers, w.experts), dtype=np.uint32)
    for l in range(w.layers):
        lg = logits(w, l, CALIB_TOKEN0 + 65536, calib_tokens)
        top = np.argpartition(-lg, w.top_k - 1, axis=1)[:, : w.top_k]
        counts[l] = np.bincount(top.ravel(), minlength=w.experts).astype(np.uint32)
    return counts


def expert_matrices(w: Workload, layer: int, expert: int):
    """(gate [I,H], up [I,H], down [H,I]) f32 weights of one expert."""
    from . import expert_weights
    return expert_weights(w.seed, layer, expert, w.hidden, w.inter, WEIGHT_SIGMA)


def layer_matrices(w: Workload, layer: int):
    """All experts of one layer: gate [E,I,H], up [E,I,H], down [E,H,I] f32."""
    from . import MAT_DOWN, MAT_GATE, MAT_UP
    g = weights(w.seed, layer, 0, w.experts, MAT_GATE, w.inter, w.hidden, WEIGHT_SIGMA)
    u = weights(w.seed, layer, 0, w.experts, MAT_UP, w.inter, w.hidden, WEIGHT_SIGMA)
    d = weights(w.seed, layer, 0, w.experts, MAT_DOWN, w.hidden, w.inter, WEIGHT_SIGMA)
    return g, u, d
