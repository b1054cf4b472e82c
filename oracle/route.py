"""Top-k softmax routing with renormalised weights (oracle, fp64).

Source: the hipfire offload explainer, opening section (a 125 GB MoE on a
32 GB card): every token activates only 8 of its layer's experts (top-8
routing), so most expert weights sit idle on any step.  The routing rule
itself is not spelled out on the pages; the reading used here is the plain
one: p = softmax(logits) over all experts, the k experts with the largest
logits are selected, and their weights are renormalised to sum to one,
w_j = p_j / sum over the selected of p.

Selection order: by logit, descending; equal logits go to the lower expert
index.  (Ordering by p or by logit is the same, since softmax is
monotonic.)  Slot j of a token holds its j-th largest selected logit.
"""
from __future__ import annotations

import numpy as np


def router_logits(x: np.ndarray, wr: np.ndarray) -> np.ndarray:
    """Router logits [T, E] = x Wr^T in fp64: x [T, H] activation values, Wr
    [E, H] router weights (hipfire offload explainer, opening section: each
    token's router picks its layer's experts; the router is the plain linear
    map of the token's hidden state, no bias)."""
    x = np.asarray(x, dtype=np.float64)
    wr = np.asarray(wr, dtype=np.float64)
    return x @ wr.T


def near_ties(logits: np.ndarray, k: int, margin) -> np.ndarray:
    """bool [T]: rows whose k-th and (k+1)-th largest logits lie within
    `margin` (scalar or [T]) of each other, where two correct computations of
    the logits (different rounding) may select different experts."""
    l = np.asarray(logits, dtype=np.float64)
    if l.shape[1] <= k:
        return np.zeros(l.shape[0], dtype=bool)
    s = -np.sort(-l, axis=1)
    return (s[:, k - 1] - s[:, k]) <= np.asarray(margin, dtype=np.float64)


def softmax(logits: np.ndarray) -> np.ndarray:
    """Row-wise softmax in fp64 with the row maximum subtracted first."""
    l = np.asarray(logits, dtype=np.float64)
    z = np.exp(l - l.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def select_topk(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices [T, k] of the k largest logits per row, by (logit desc, index asc)."""
    l = np.asarray(logits, dtype=np.float64)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError(f"k={k} must be in [1, E={E}]")
    out = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        order = np.lexsort((idx, -l[t]))   # primary key: -logit; secondary: index
        out[t] = order[:k]
    return out


def route(logits: np.ndarray, k: int):
    """(idx int32 [T,k], wts f64 [T,k]): top-k experts and renormalised weights."""
    p = softmax(logits)
    idx = select_topk(logits, k)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    return idx, sel / sel.sum(axis=1, keepdims=True)


def group_by_expert(idx: np.ndarray, n_experts: int):
    """Group the (token, slot) pairs by expert.

    Returns cnt int32 [E] (pairs per expert), off int32 [E+1] (exclusive prefix
    sum of cnt) and perm int32 [T*k]: for expert e, perm[off[e]:off[e+1]] are
    the flat pair ids t*k + j with idx[t, j] == e, in increasing order."""
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    cnt = np.zeros(n_experts, dtype=np.int32)
    buckets = [[] for _ in range(n_experts)]
    for pair, e in enumerate(flat):
        buckets[e].append(pair)
        cnt[e] += 1
    off = np.zeros(n_experts + 1, dtype=np.int32)
    off[1:] = np.cumsum(cnt)
    perm = np.array([p for b in buckets for p in b], dtype=np.int32)
    return cnt, off, perm
