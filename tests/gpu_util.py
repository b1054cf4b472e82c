"""Helpers for the GPU tests: device models from the seeded generators, and
oracle-side views of the same experts (regenerated on the host and packed by
the oracle, never taken from the CUDA path)."""
import numpy as np

import synth
from synth import workloads as W

TOL = 1e-3        # max relative error of y per token, fp32 accumulation


def max_rel_err(y, ref):
    """max_i |y_i - r_i| / max_i |r_i| per row, then the max over rows."""
    y = np.asarray(y, np.float64).reshape(-1, ref.shape[-1])
    r = np.asarray(ref, np.float64).reshape(-1, ref.shape[-1])
    return float(np.max(np.max(np.abs(y - r), axis=1) / np.max(np.abs(r), axis=1)))


def device_fill(torch, w):
    """fill(layer, g, u, d) writing workload w's f32 weights on the GPU."""
    def fill(l, g, u, d):
        s = torch.cuda.current_stream().cuda_stream
        E = g.shape[0]
        synth.weights_dev(g.data_ptr(), w.seed, l, 0, E, synth.MAT_GATE, w.inter, w.hidden,
                          W.WEIGHT_SIGMA, s)
        synth.weights_dev(u.data_ptr(), w.seed, l, 0, E, synth.MAT_UP, w.inter, w.hidden,
                          W.WEIGHT_SIGMA, s)
        synth.weights_dev(d.data_ptr(), w.seed, l, 0, E, synth.MAT_DOWN, w.hidden, w.inter,
                          W.WEIGHT_SIGMA, s)
    return fill


class OraclePackedLayer:
    """Experts of one layer, regenerated on the host and packed by the oracle on
    first use (behaves like a uint8 [E, expert_bytes] array for the oracle)."""

    def __init__(self, w, layer):
        from oracle import hfq4
        self.w, self.layer, self._hfq4 = w, layer, hfq4
        self._cache = {}

    def __len__(self):
        return self.w.experts

    def __getitem__(self, e):
        e = int(e)
        if e not in self._cache:
            g, u, d = W.expert_matrices(self.w, self.layer, e)
            self._cache[e] = self._hfq4.pack_expert(g, u, d)
        return self._cache[e]
