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


# ------------------------------------------------------------ error report

_REPORT = []


def elementwise_errors(y, ref):
    """Elementwise relative errors |y_i - r_i| / max(|r_i|, 1e-6 * max_j |r_j|),
    the floor taken per token row; returns the median and the maximum beside
    the normwise metric of max_rel_err."""
    y = np.asarray(y, np.float64).reshape(-1, ref.shape[-1])
    r = np.asarray(ref, np.float64).reshape(-1, ref.shape[-1])
    floor = 1e-6 * np.max(np.abs(r), axis=1, keepdims=True)
    e = np.abs(y - r) / np.maximum(np.abs(r), floor)
    return {"normwise": max_rel_err(y, r), "elem_median": float(np.median(e)),
            "elem_max": float(np.max(e))}


def report(y, ref, name=None):
    """Records the errors of one parity comparison under the running test's
    name (printed at the end of the pytest run) and returns the normwise error
    the tests assert on."""
    import os
    d = elementwise_errors(y, ref)
    name = name or os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0].split("::")[-1]
    _REPORT.append((name, d))
    return d["normwise"]


def report_lines():
    return [f"{n}: normwise {d['normwise']:.3e}  elementwise median {d['elem_median']:.3e}  "
            f"max {d['elem_max']:.3e}" for n, d in _REPORT]


# ------------------------------------------- oracle on many tokens, by expert

def _expert_rows(args):
    """One expert's FFN outputs for a batch of token rows (worker process)."""
    from oracle import moe
    w, layer, e, x_bits, tc = args
    cache = moe.ExpertCache(OraclePackedLayer(w, layer), w.hidden, w.inter, tc=tc)
    x = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    return e, moe.expert_ffn(*cache(e), x)


def oracle_rows(w, layer, x_bits, idx, wts, tokens, tc=False, workers=None):
    """y [len(tokens), H] (fp64) of the oracle's routed layer for the listed
    tokens of a large batch, computed expert by expert so that one expert's
    fp64 weights are alive per worker at a time: every (token, slot) pair of
    the listed tokens runs moe.expert_ffn of its expert, and y_t is the sum of
    w_tj * o_tj over the slots (fp64, the terms of moe.moe_layer); tc=True
    takes the tensor-core model's weights.  Workers are spawned processes (the
    calling process may hold a CUDA context); workers=0 runs in this process."""
    import multiprocessing as mp
    import os
    tokens = np.asarray(tokens, np.int64)
    k = idx.shape[1]
    by_e = {}
    for i, t in enumerate(tokens):
        for j in range(k):
            by_e.setdefault(int(idx[t, j]), []).append((i, j))
    jobs = [(w, layer, e, np.ascontiguousarray(x_bits[tokens[[i for i, _ in pr]]]), tc)
            for e, pr in sorted(by_e.items())]
    y = np.zeros((len(tokens), w.hidden))

    def take(e, o):
        for r, (i, j) in enumerate(by_e[e]):
            y[i] += float(wts[tokens[i], j]) * o[r]

    if workers == 0:
        for job in jobs:
            take(*_expert_rows(job))
    else:
        n = workers or max(1, min(32, os.cpu_count() or 1))
        with mp.get_context("spawn").Pool(n) as pool:
            for res in pool.imap_unordered(_expert_rows, jobs):
                take(*res)
    return y
