"""Expert placement between HBM and pinned host memory (oracle).

Source: the hipfire offload explainer, section "placement algorithm":
  1. auto (the default): after the backbone, routed experts are placed layer
     by layer until the VRAM budget is used up; the remaining layers go to
     pinned host memory (fit-capacity placement);
  2. a manual knob N: the experts of the first N layers stay in VRAM, layers
     N onwards go to host memory;
  3. an expert hot set ranked by decode heat makes VRAM go to the most
     activated experts first;
  4. a configuration that does not fit is refused at load, naming the byte
     deficit rather than failing later.
Section "PCIe pass-through" of the same page: host-mapped experts are read by
the GPU kernel directly over PCIe.

Readings where the page is silent (stated, not the page's):
  * the hot set of a host layer is its top-h experts by calibration selection
    count, ties to the lower expert index; they are placed in HBM;
  * the budget covers expert bytes only (no backbone in this scope);
  * auto picks the largest N such that N full layers plus the hot sets of the
    L-N host layers fit: need(N) = (N*E + (L-N)*h) * expert_bytes;
  * slots number the experts of each location in (layer, expert) order.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

HBM, HOST = 0, 1


@dataclass
class Placement:
    ok: bool
    resident_layers: int
    loc: np.ndarray        # uint8 [L, E]: 0 = HBM, 1 = host
    slot: np.ndarray       # int64 [L, E]: index within its location's arena
    hbm_needed: int
    host_needed: int
    deficit: int           # bytes missing from the budget when not ok


def hot_experts(counts_row: np.ndarray, h: int) -> np.ndarray:
    """Top-h experts of one layer by (count desc, index asc)."""
    E = len(counts_row)
    order = sorted(range(E), key=lambda e: (-int(counts_row[e]), e))
    return np.array(sorted(order[:h]), dtype=np.int64)


def need_bytes(L: int, E: int, n: int, h: int, expert_bytes: int) -> int:
    return (n * E + (L - n) * min(h, E)) * expert_bytes


def place(counts: np.ndarray, expert_bytes: int, resident_layers: int, hot_per_layer: int,
          hbm_budget: int) -> Placement:
    counts = np.asarray(counts)
    L, E = counts.shape
    h = min(max(hot_per_layer, 0), E)
    if resident_layers < 0:
        n = -1
        for cand in range(L, -1, -1):
            if need_bytes(L, E, cand, h, expert_bytes) <= hbm_budget:
                n = cand
                break
        if n < 0:
            need = need_bytes(L, E, 0, h, expert_bytes)
            return Placement(False, 0, np.zeros((L, E), np.uint8), np.zeros((L, E), np.int64),
                             need, L * E * expert_bytes - need, need - hbm_budget)
    else:
        if resident_layers > L:
            raise ValueError("resident_layers > layers")
        n = resident_layers
    loc = np.full((L, E), HOST, dtype=np.uint8)
    loc[:n] = HBM
    for l in range(n, L):
        loc[l, hot_experts(counts[l], h)] = HBM
    slot = np.zeros((L, E), dtype=np.int64)
    next_slot = {HBM: 0, HOST: 0}
    for l in range(L):
        for e in range(E):
            slot[l, e] = next_slot[int(loc[l, e])]
            next_slot[int(loc[l, e])] += 1
    hbm_needed = next_slot[HBM] * expert_bytes
    host_needed = next_slot[HOST] * expert_bytes
    ok = hbm_needed <= hbm_budget
    return Placement(ok, n, loc, slot, hbm_needed, host_needed, max(0, hbm_needed - hbm_budget))
