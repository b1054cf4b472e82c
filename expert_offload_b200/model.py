"""Expert storage: pack a model's experts into HBM and/or a pinned host arena
and build the per-layer pointer tables the kernels read.

This is the loader/placer of the pages (hipfire offload explainer, "placement
algorithm": layers 0..N-1 resident, later layers host-mapped, the hot set of
each host layer resident; Strata report, "model and engine": a per-(layer,
expert) table locates every expert).  torch provides the device memory; the
quantisation and placement run in the library.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import (HfqError, Layer, hfq4_expert_bytes, hfq4_pack_experts_device,
               hfq_host_arena_create, hfq_host_arena_destroy, hfq_placement_build,
               hfq_placement_pointers)


class ExpertStore:
    """Packed experts of L layers x E experts, each at a placement-chosen slot.

    fill(layer, gate, up, down) must write f32 weights into the given device
    tensors (gate/up [E, I, H], down [E, H, I]) for every expert of a layer.
    loc: uint8 [L, E] (0 = HBM, 1 = host) or None for all-HBM.
    """

    def __init__(self, torch, layers: int, experts: int, hidden: int, inter: int, fill,
                 loc=None, slot=None, device="cuda", chunk_experts: int = 64,
                 hugepage: bool = False):
        self.torch = torch
        self.L, self.E, self.H, self.I = layers, experts, hidden, inter
        self.eb = hfq4_expert_bytes(hidden, inter)
        if loc is None:
            loc = np.zeros((layers, experts), np.uint8)
            slot = np.arange(layers * experts, dtype=np.int64).reshape(layers, experts)
        self.loc, self.slot = np.ascontiguousarray(loc, np.uint8), np.ascontiguousarray(slot)
        n_hbm = int((self.loc == 0).sum())
        n_host = int((self.loc == 1).sum())
        self.hbm = torch.empty(max(n_hbm, 1) * self.eb, dtype=torch.uint8, device=device)
        self.host_ptr = self.host_dev = None
        self.host_view = None
        if n_host:
            self.host_ptr, self.host_dev = hfq_host_arena_create(n_host * self.eb,
                                                                 1 if hugepage else 0)
            buf = (ctypes.c_uint8 * (n_host * self.eb)).from_address(self.host_ptr)
            self.host_view = torch.from_numpy(np.frombuffer(buf, dtype=np.uint8))
        ptrs = hfq_placement_pointers(self.loc, self.slot, self.eb, self.hbm.data_ptr(),
                                      self.host_dev or 0)
        self.ptr_table = torch.from_numpy(ptrs.view(np.int64)).to(device)
        self.loc_table = torch.from_numpy(self.loc).to(device)
        self._pack_all(fill, device, chunk_experts)
        self.layers = [Layer(self.ptr_table[l], experts, hidden, inter,
                             expert_loc=self.loc_table[l] if n_host else None)
                       for l in range(layers)]

    def _pack_all(self, fill, device, chunk):
        torch = self.torch
        E, H, I, eb = self.E, self.H, self.I, self.eb
        g = torch.empty((E, I, H), dtype=torch.float32, device=device)
        u = torch.empty((E, I, H), dtype=torch.float32, device=device)
        d = torch.empty((E, H, I), dtype=torch.float32, device=device)
        staging = torch.empty(E * eb, dtype=torch.uint8, device=device)
        for l in range(self.L):
            fill(l, g, u, d)
            hfq4_pack_experts_device(g, u, d, staging, E, H, I)
            for e in range(E):
                dst_slot = int(self.slot[l, e])
                src = staging[e * eb:(e + 1) * eb]
                if self.loc[l, e] == 0:
                    self.hbm[dst_slot * eb:(dst_slot + 1) * eb].copy_(src)
                else:
                    self.host_view[dst_slot * eb:(dst_slot + 1) * eb].copy_(src)
        torch.cuda.synchronize()
        del g, u, d, staging

    def expert_bytes_at(self, layer: int, expert: int):
        """This expert's packed bytes as a numpy array (copied to the host)."""
        s = int(self.slot[layer, expert])
        if self.loc[layer, expert] == 0:
            return self.hbm[s * self.eb:(s + 1) * self.eb].cpu().numpy()
        return self.host_view[s * self.eb:(s + 1) * self.eb].numpy().copy()

    def close(self):
        if self.host_ptr:
            self.host_view = None
            hfq_host_arena_destroy(self.host_ptr)
            self.host_ptr = None

    def __del__(self):
        try:
            self.close()
        except (HfqError, AttributeError, TypeError):
            pass


def place(counts, expert_bytes: int, resident_layers: int, hot_per_layer: int, hbm_budget: int):
    """Placement through the library (loud refusal raises HfqError)."""
    loc, slot, hn, hs = hfq_placement_build(counts, expert_bytes, resident_layers, hot_per_layer,
                                            hbm_budget)
    return loc, slot, hn, hs
