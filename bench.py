#!/usr/bin/env python
"""Benchmark of the routed-expert HFQ4 MoE layer on B200.

Headline workload: the decode stack of 40 MoE layers (hidden 2048, expert
intermediate 512, 256 experts per layer, top-8, 1 token, bf16 residual
stream), all experts resident in HBM.  A step is one token through all 40
layers: route, gate/up GEMV with SiLU*up, down GEMV with the weighted
combine, residual add.  Every step routes a different token (64 distinct
tokens' logits cycled), so a step streams 535 MB of expert weights, more
than the 126 MB L2: no flush is needed between steps.

The default run (no --workload) also measures, in the same process and on
the same GPU, the other workloads of the layer and reports each under
"workloads" with its own roofline and clocks:
  * verify stack: 48 layers x 512 experts, skewed routing, 1/2/5/8 tokens;
  * offload sweep: the 48 x 512 model with layers N..47 read zero-copy from
    pinned host memory, N in {48, 36, 24, 13, 0}, 0 or 51 hot experts per
    host layer kept in HBM;
  * prefill chunks: one 512-expert layer, 512/2048/8192 tokens with Zipf(1.1)
    popularity, tensor-core path and GEMV path.
Beside them: a read-only HBM stream and the PCIe link measured on the box,
and the oracle timed on the host's cores (one core, then one process per
core).

Prints one JSON line (rank 0).  --impl reference times the oracle (CPU,
fp64) on bounded samples of the headline workload instead.
"""
from __future__ import annotations

import os

# The oracle legs run single-threaded: BLAS thread pools are sized when numpy
# loads, so they are pinned to one thread before anything imports it (and
# checked with threadpoolctl before any oracle timing).
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS", "BLIS_NUM_THREADS",
           "VECLIB_MAXIMUM_THREADS", "NUMEXPR_NUM_THREADS"):
    os.environ[_v] = "1"

import argparse  # noqa: E402
import json  # noqa: E402
import statistics  # noqa: E402
import subprocess  # noqa: E402
import sys  # noqa: E402
import tempfile  # noqa: E402
import time  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s and achieved GB/s as % of HBM/PCIe roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
SPEC_HBM_GBS = 8000.0          # the B200 HBM3e figure the layer's roofline is quoted against


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "verify", "offload", "prefill", "routed"], default=None,
                    help="one workload alone (default: the headline decode stack plus all others)")
    ap.add_argument("--no-suite", action="store_true", help="the headline workload only")
    ap.add_argument("--tokens", type=int, default=8, help="tokens per step (verify, prefill)")
    ap.add_argument("--resident-layers", type=int, default=None, help="offload: N")
    ap.add_argument("--hot", type=int, default=0, help="offload: hot experts per host layer")
    ap.add_argument("--hugepage", action="store_true",
                    help="offload: host arena on 2 MiB transparent huge pages (madvise)")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--distinct-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="oracle time per CPU baseline figure")
    ap.add_argument("--path", type=int, default=0, help="0 auto, 1 GEMV")
    ap.add_argument("--layers", type=int, default=None,
                    help="a prefix of the stack (small profiling cases)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured bf16 burst"
    return FALLBACK_BF16_TFLOPS, "fallback bf16"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        sm, smax, reasons = [], [], set()
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ link probes

def measure_pcie(torch, eo, nbytes=1 << 30, flags=0):
    """Host-to-device bandwidth two ways: a pinned cudaMemcpy and the zero-copy
    read kernel over a mapped arena (the strata report's link probe, done here
    with the expert kernel's own load path)."""
    h, d = eo.hfq_host_arena_create(nbytes, flags)
    try:
        sink = torch.zeros(1, dtype=torch.int64, device="cuda")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        eo.hfq_probe_read(d, nbytes, 1, sink)
        torch.cuda.synchronize()
        e0.record()
        eo.hfq_probe_read(d, nbytes, 2, sink)
        e1.record()
        torch.cuda.synchronize()
        zc = 2 * nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9
        import ctypes

        import numpy as np
        buf = (ctypes.c_uint8 * nbytes).from_address(h)
        src = torch.from_numpy(np.frombuffer(buf, dtype=np.uint8))
        dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        dst.copy_(src, non_blocking=True)
        torch.cuda.synchronize()
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        cp = nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9
    finally:
        eo.hfq_host_arena_destroy(h)
    return {"zero_copy_read_gbs": round(zc, 2), "pinned_memcpy_gbs": round(cp, 2)}


def measure_hbm_read(torch, eo, nbytes=4 << 30):
    """Read-only stream over a buffer far larger than L2 (the probe kernel's
    16-byte loads), best of three launches."""
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    eo.hfq_probe_read(buf, nbytes, 1, sink)
    best = 0.0
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        eo.hfq_probe_read(buf, nbytes, 2, sink)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, 2 * nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9)
    del buf
    return round(best, 1)


def max_over_ranks(dist, values, device):
    """Each value's maximum over all ranks (a replicated job takes as long as
    its slowest rank); the values unchanged without a process group."""
    if dist is None:
        return [float(v) for v in values]
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_rate(world, steps, units_per_step, job_ms):
    """Whole-job throughput: the units all `world` replicas processed in
    `steps` steps, over the job's time."""
    return world * steps * units_per_step / (job_ms / 1e3)


# ------------------------------------------------------- stacks (T <= 8)

def step_bytes(logits_g, k, eb, loc):
    """(HBM bytes, host bytes) one step streams: every unique selected expert of
    every layer once (router logits and activations, < 0.1 %, not counted)."""
    import numpy as np
    hbm = host = 0
    for l in range(logits_g.shape[0]):
        top = np.argpartition(-logits_g[l], k - 1, axis=1)[:, :k]
        for e in np.unique(top):
            if loc is not None and loc[l, e]:
                host += eb
            else:
                hbm += eb
    return hbm, host


def fill_for(torch, synth, W, w):
    def fill(l, g, u, d):
        s = torch.cuda.current_stream().cuda_stream
        E, H, I = w.experts, w.hidden, w.inter
        synth.weights_dev(g.data_ptr(), w.seed, l, 0, E, synth.MAT_GATE, I, H, W.WEIGHT_SIGMA, s)
        synth.weights_dev(u.data_ptr(), w.seed, l, 0, E, synth.MAT_UP, I, H, W.WEIGHT_SIGMA, s)
        synth.weights_dev(d.data_ptr(), w.seed, l, 0, E, synth.MAT_DOWN, H, I, W.WEIGHT_SIGMA, s)
    return fill


class StackInputs:
    """G token groups of a stack workload: logits [G, L, T, E] and inputs
    [G, T, H] (bf16), on the device, plus each group's streamed bytes."""

    def __init__(self, torch, W, w, L, T, G, token0=0):
        import numpy as np
        # one generator call per layer for all G * T tokens (token g * T + t of
        # group g), the same values as per-group calls
        lg = np.stack([W.logits(w, l, token0, G * T) for l in range(L)])       # [L, G*T, E]
        self.logits = np.ascontiguousarray(lg.reshape(L, G, T, -1).transpose(1, 0, 2, 3))
        self.xs = W.activations(w, token0, G * T)[0].reshape(G, T, -1)
        self.d_logits = torch.from_numpy(self.logits).cuda()
        self.d_x = torch.from_numpy(self.xs.view(np.int16)).cuda()
        self.G, self.T = G, T


class StackTimer:
    """CUDA graphs of one stack launch per token group, replayed back to back
    on one stream with an event after each launch."""

    def __init__(self, torch, eo, layers, inp, k, H, I, E, path=0, router=None):
        self.torch, self.eo, self.inp, self.k = torch, eo, inp, k
        self.router = router
        T, G = inp.T, inp.G
        self.layers = layers
        self.arr = eo.layer_array(layers)
        self.ws = torch.zeros(eo.hfq4_stack_workspace_bytes(T, k, H, I, E), dtype=torch.uint8,
                              device="cuda")
        self.x_out = torch.empty((G, T, H), dtype=torch.int16, device="cuda")
        self.stream = torch.cuda.Stream()
        self.path = path
        with torch.cuda.stream(self.stream):
            for g in range(G):
                self.step(g)
        torch.cuda.synchronize()
        eo.hfq_workspace_status(self.ws, self.stream)
        self.graphs = []
        try:
            for g in range(G):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=self.stream):
                    self.step(g)
                self.graphs.append(gr)
            torch.cuda.synchronize()
            self.replay = [gr.replay for gr in self.graphs]
            self.launch_mode = "cuda graph per token group"
        except RuntimeError as exc:          # capture not possible: launch directly
            print(f"graph capture failed ({exc}); launching directly", file=sys.stderr)
            torch.cuda.synchronize()
            self.graphs = []
            self.replay = [(lambda g=g: self.step(g)) for g in range(G)]
            self.launch_mode = "direct launch"

    def step(self, g):
        if self.router is not None:
            self.eo.hfq4_moe_decode_stack_routed(self.layers, self.router, self.eo.HFQ_BF16, self.k,
                                                 self.inp.d_x[g], self.inp.T, self.x_out[g],
                                                 self.ws, stream=self.stream,
                                                 _layer_array=self.arr)
            return
        self.eo.hfq4_moe_decode_stack(self.layers, self.inp.d_logits[g], self.k, self.inp.d_x[g],
                                      self.inp.T, self.x_out[g], self.ws, path=self.path,
                                      stream=self.stream, _layer_array=self.arr)

    def run(self, K, W, dist=None, gpu=0):
        """(total ms, per-launch ms list, clocks) of K timed launches after W."""
        torch = self.torch
        G = self.inp.G
        with torch.cuda.stream(self.stream):
            for i in range(W):
                self.replay[i % G]()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        sampler = ClockSampler(gpu)
        sampler.start()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        with torch.cuda.stream(self.stream):
            ev[0].record(self.stream)
            for i in range(K):
                self.replay[i % G]()
                ev[i + 1].record(self.stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        clocks = sampler.stop()
        self.eo.hfq_workspace_status(self.ws, self.stream)
        return (ev[0].elapsed_time(ev[K]), [ev[i].elapsed_time(ev[i + 1]) for i in range(K)], clocks)

    def close(self):
        self.graphs = []
        self.replay = []


def kernel_name(T, launches):
    if launches != 1:
        return "per-layer route + gate/up + down launches"
    return ("decode1_kernel" if T == 1 else "verify_kernel") + \
        " (persistent: all layers of one step per launch)"


def hbm_roofline(bytes_per_step, mean_launch_ms, peak, peak_kind, read_gbs, kernel):
    achieved = bytes_per_step / (mean_launch_ms / 1e3) / 1e9
    r = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
         "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} copy (MEASURED_PEAKS.json)",
         "kernel": kernel, "bytes_per_launch": round(bytes_per_step),
         "mean_launch_ms": round(mean_launch_ms, 5),
         "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4)}
    if read_gbs:
        r["hbm_read_stream_gbs"] = read_gbs
        r["frac_of_read_stream"] = round(achieved / read_gbs, 4)
    return r


def offload_roofline(logits, k, eb, loc, hbm_b, host_b, mean_launch_ms, peak, peak_kind, bw_pcie,
                     pcie, kernel):
    """Per layer the HBM and PCIe streams overlap: the roofline time of a step
    is the sum over layers of max(HBM bytes / HBM rate, host bytes / PCIe rate)."""
    G, L = logits.shape[0], logits.shape[1]
    roof_ms = 0.0
    for g in range(G):
        for l in range(L):
            hb, hs = step_bytes(logits[g, l:l + 1], k, eb, loc[l:l + 1])
            roof_ms += max(hb / (peak * 1e9), hs / (bw_pcie * 1e9)) * 1e3
    roof_ms /= G
    return {"bound": "pcie" if host_b > 0 else "hbm",
            "achieved": round((hbm_b + host_b) / (mean_launch_ms / 1e3) / 1e9, 2),
            "peak": round((hbm_b + host_b) / (roof_ms / 1e3) / 1e9, 2), "unit": "GB/s",
            "frac": round(roof_ms / mean_launch_ms, 4), "kernel": kernel,
            "peak_source": f"roofline time from the measured PCIe {bw_pcie} GB/s and the "
                           f"{peak_kind} HBM {peak} GB/s, per layer",
            "hbm_bytes_per_launch": round(hbm_b), "host_bytes_per_launch": round(host_b),
            "host_gbs_achieved": round(host_b / (mean_launch_ms / 1e3) / 1e9, 2),
            "pcie": pcie, "mean_launch_ms": round(mean_launch_ms, 5)}


def sub_result(T, K, total_ms, per_launch, clocks, roofline, launches, extra=None):
    mean_ms = sum(per_launch) / K
    d = {"value": round(K * T / (total_ms / 1e3), 2), "unit": "tokens/s",
         "ms_per_step": round(total_ms / K, 5), "steps": K, "tokens_per_step": T,
         "gpu_launches": launches * K, "roofline": roofline, "clocks": clocks}
    if extra:
        d.update(extra)
    return d


# ------------------------------------------------------------- the headline

def run_headline(args, rank, world, local_rank, dist):
    """The decode stack (or the workload --workload names), timed on the device
    and end to end through the C ABI."""
    import numpy as np
    import torch

    import expert_offload_b200 as eo
    import synth
    from expert_offload_b200.model import ExpertStore
    from synth import workloads as W

    wl = args.workload or "decode"
    w = W.WORKLOADS[{"decode": 2, "verify": 3, "offload": 5}[wl]]
    if args.layers:
        import dataclasses
        w = dataclasses.replace(w, layers=args.layers, name=f"{w.name} (first {args.layers} layers)")
    T = args.tokens if wl == "verify" else 1
    L, H, I, E, k = w.layers, w.hidden, w.inter, w.experts, w.top_k
    eb = eo.hfq4_expert_bytes(H, I)
    G = args.distinct_tokens
    loc = slot = place_info = None
    if wl == "offload":
        counts = W.calibration_counts(w, 1024)
        N = w.layers if args.resident_layers is None else args.resident_layers
        loc, slot, hn, hs = eo.hfq_placement_build(counts, eb, N, args.hot, 170 * 2**30)
        place_info = {"resident_layers": N, "hot_per_layer": args.hot, "hbm_bytes": hn,
                      "host_bytes": hs, "hugepage": bool(args.hugepage)}
    store = ExpertStore(torch, L, E, H, I, fill_for(torch, synth, W, w), loc=loc, slot=slot,
                        hugepage=args.hugepage)
    inp = StackInputs(torch, W, w, L, T, G)
    per_group = [step_bytes(inp.logits[g], k, eb, loc) for g in range(G)]
    timer = StackTimer(torch, eo, store.layers, inp, k, H, I, E, path=args.path)
    launches = eo.hfq4_stack_launches(L, T, k, H, I)
    K = args.steps
    total_ms, per_launch, clocks = timer.run(K, args.warmup, dist, local_rank)

    # end to end through the C ABI: pinned host inputs copied in, result copied out
    K2 = min(args.e2e_steps, K)
    h_logits = torch.from_numpy(inp.logits).pin_memory()
    h_x = torch.from_numpy(inp.xs.view(np.int16)).pin_memory()
    h_out = torch.empty((G, T, H), dtype=torch.int16).pin_memory()
    in_l = torch.empty_like(inp.d_logits[0])
    in_x = torch.empty_like(inp.d_x[0])
    out_x = torch.empty_like(timer.x_out[0])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = timer.stream

    def e2e_step(i):
        g = i % G
        in_l.copy_(h_logits[g], non_blocking=True)
        in_x.copy_(h_x[g], non_blocking=True)
        eo.hfq4_moe_decode_stack(store.layers, in_l, k, in_x, T, out_x, timer.ws, path=args.path,
                                 stream=stream, _layer_array=timer.arr)
        h_out[g].copy_(out_x, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(min(20, K2)):
            e2e_step(i)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(K2):
            e2e_step(i)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    eo.hfq_workspace_status(timer.ws, stream)
    total_ms, e2e_ms = max_over_ranks(dist, [total_ms, e2e_ms], "cuda")

    hbm_b = sum(per_group[i % G][0] for i in range(K)) / K
    host_b = sum(per_group[i % G][1] for i in range(K)) / K
    mean_launch_ms = sum(per_launch) / K
    peak, peak_kind = peaks()
    read_gbs = measure_hbm_read(torch, eo)
    out = {
        "metric": METRIC, "value": round(job_rate(world, K, T, total_ms), 2), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "layers": L, "hidden": H, "inter": I, "experts": E,
                   "top_k": k, "tokens_per_step": T, "weights": "hfq4 (136-byte blocks)",
                   "activations": "bf16", "accumulate": "f32",
                   "distinct_token_groups_cycled": G,
                   "expert_bytes_per_step": round(hbm_b + host_b),
                   "launch": timer.launch_mode,
                   "l2": "per-step working set > 126 MB L2 (every step routes new tokens); "
                         "no flush",
                   "parallelism": f"replicas x{world}"},
        "gpu_launches": launches * K,
        "clocks": clocks,
    }
    kernel = kernel_name(T, launches)
    if wl == "offload":
        pcie = measure_pcie(torch, eo)
        out["config"]["placement"] = place_info
        out["roofline"] = offload_roofline(inp.logits, k, eb, loc, hbm_b, host_b, mean_launch_ms,
                                           peak, peak_kind, max(pcie.values()), pcie, kernel)
    else:
        out["roofline"] = hbm_roofline(hbm_b + host_b, mean_launch_ms, peak, peak_kind, read_gbs,
                                       kernel)
        # DRAM bytes (read + write) per decode1_kernel launch from an ncu capture of
        # the first 10 layers of this workload, scaled by 4 to the 40 layers (the
        # per-layer work is the same); None once the kernel has changed since
        traffic = TRAFFIC_DECODE_L40 if (wl == "decode" and L == 40 and not args.layers) else None
        out["roofline"]["traffic"] = traffic
        out["roofline"]["traffic_source"] = TRAFFIC_SOURCE if traffic else None
    out["e2e"] = {"value": round(job_rate(world, K2, T, e2e_ms), 2), "unit": "tokens/s",
                  "h2d_bytes_per_step": int(in_l.numel() * 4 + in_x.numel() * 2),
                  "d2h_bytes_per_step": int(out_x.numel() * 2)}
    timer.close()
    store.close()
    del store, timer, inp
    torch.cuda.empty_cache()
    return out, w


# DRAM traffic of one decode1_kernel launch on the headline workload, or None
# while no capture of the current kernel exists (see profiles/).
TRAFFIC_DECODE_L40 = 4 * (133837056 + 2886144)
TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one decode1_kernel<0, 1, 0> launch "
                  "over the first 10 layers (133,837,056 + 2,886,144 B), x 4")


# --------------------------------------------------------- the other configs

def run_routed(args, K, W_):
    """The decode stack with each layer's router in the loop (bf16 Wr, one
    launch per token): the logits come from the residual stream, so the
    experts a step reads are known only inside the launch; with one token
    every layer reads exactly k distinct experts plus its router matrix."""
    import numpy as np
    import torch

    import expert_offload_b200 as eo
    import synth
    from expert_offload_b200.model import ExpertStore
    from synth import workloads as W

    w = W.WORKLOADS[2]
    L, H, I, E, k, T = w.layers, w.hidden, w.inter, w.experts, w.top_k, 1
    eb = eo.hfq4_expert_bytes(H, I)
    store = ExpertStore(torch, L, E, H, I, fill_for(torch, synth, W, w))
    wr = np.stack([W.router_weights(w, l) for l in range(L)])
    router = torch.from_numpy(synth.to_bf16_bits(wr).view(np.int16)).cuda()
    inp = StackInputs(torch, W, w, 1, T, args.distinct_tokens)      # x0 per token; logits unused
    timer = StackTimer(torch, eo, store.layers, inp, k, H, I, E, router=router)
    total_ms, per_launch, clocks = timer.run(K, W_)
    launches = eo.hfq4_stack_launches(L, T, k, H, I)
    bytes_step = L * (k * eb + E * H * 2)
    peak, peak_kind = peaks()
    roof = hbm_roofline(bytes_step, sum(per_launch) / K, peak, peak_kind, None,
                        kernel_name(T, launches) + ", router fused")
    res = {"decode_routed": sub_result(
        T, K, total_ms, per_launch, clocks, roof, launches,
        {"workload": w.name + ", bf16 router in the loop",
         "bytes_per_step": "L * (k distinct experts + the E x H bf16 router matrix)"})}
    timer.close()
    store.close()
    del store, timer, router
    torch.cuda.empty_cache()
    return res


def run_verify_suite(args, K, W_):
    """48 x 512 experts, skewed routing, T = 1, 2, 5, 8 (one model, four runs)."""
    import torch

    import expert_offload_b200 as eo
    import synth
    from expert_offload_b200.model import ExpertStore
    from synth import workloads as W

    w = W.WORKLOADS[3]
    L, H, I, E, k = w.layers, w.hidden, w.inter, w.experts, w.top_k
    eb = eo.hfq4_expert_bytes(H, I)
    peak, peak_kind = peaks()
    store = ExpertStore(torch, L, E, H, I, fill_for(torch, synth, W, w))
    res = {}
    for T in (1, 2, 5, 8):
        inp = StackInputs(torch, W, w, L, T, 16)
        per_group = [step_bytes(inp.logits[g], k, eb, None) for g in range(inp.G)]
        timer = StackTimer(torch, eo, store.layers, inp, k, H, I, E)
        total_ms, per_launch, clocks = timer.run(K, W_)
        hbm_b = sum(per_group[i % inp.G][0] for i in range(K)) / K
        launches = eo.hfq4_stack_launches(L, T, k, H, I)
        roof = hbm_roofline(hbm_b, sum(per_launch) / K, peak, peak_kind, None,
                            kernel_name(T, launches))
        res[f"verify_t{T}"] = sub_result(T, K, total_ms, per_launch, clocks, roof, launches,
                                         {"workload": w.name, "tokens_per_step": T})
        timer.close()
    store.close()
    del store
    torch.cuda.empty_cache()
    return res


def thp_state():
    """The kernel's transparent-huge-page mode and the anonymous huge pages in
    use now (kB), as the system reports them."""
    out = {}
    try:
        out["mode"] = open("/sys/kernel/mm/transparent_hugepage/enabled").read().strip()
    except OSError:
        out["mode"] = "unknown"
    try:
        for line in open("/proc/meminfo"):
            if line.startswith("AnonHugePages:"):
                out["anon_huge_kb"] = int(line.split()[1])
    except OSError:
        pass
    return out


class DualModel:
    """Every expert of a model twice: packed in HBM and in one pinned, mapped
    host arena, at the same offset (layer * E + expert) * expert_bytes.  A
    placement then only chooses, per (layer, expert), which copy the kernels'
    pointer table names; no bytes move between placements."""

    def __init__(self, torch, eo, store, hugepage=False):
        import ctypes

        import numpy as np
        self.torch, self.eo, self.store = torch, eo, store
        L, E, eb = store.L, store.E, store.eb
        self.host, self.host_dev = eo.hfq_host_arena_create(L * E * eb, 1 if hugepage else 0)
        buf = (ctypes.c_uint8 * (L * E * eb)).from_address(self.host)
        view = torch.from_numpy(np.frombuffer(buf, dtype=np.uint8))
        chunk = 1 << 30
        for o in range(0, L * E * eb, chunk):
            n = min(chunk, L * E * eb - o)
            view[o:o + n].copy_(store.hbm[o:o + n])
        torch.cuda.synchronize()
        self.slot = np.arange(L * E, dtype=np.int64).reshape(L, E)

    def layers(self, loc):
        import numpy as np
        eo, torch, s = self.eo, self.torch, self.store
        ptrs = eo.hfq_placement_pointers(loc, self.slot, s.eb, s.hbm.data_ptr(), self.host_dev)
        self._ptr = torch.from_numpy(ptrs.view(np.int64)).cuda()
        self._loc = torch.from_numpy(np.ascontiguousarray(loc, np.uint8)).cuda()
        return [eo.Layer(self._ptr[l], s.E, s.H, s.I, expert_loc=self._loc[l]) for l in range(s.L)]

    def close(self):
        if self.host:
            self.eo.hfq_host_arena_destroy(self.host)
            self.host = None


def run_offload_suite(args, K, W_):
    """The 48 x 512 model, 1 token, layers N..47 host-mapped, N in {48, 36, 24,
    13, 0}, with 0 and 51 hot experts per host layer in HBM."""
    import torch

    import expert_offload_b200 as eo
    import synth
    from expert_offload_b200.model import ExpertStore
    from synth import workloads as W

    w = W.WORKLOADS[5]
    L, H, I, E, k = w.layers, w.hidden, w.inter, w.experts, w.top_k
    eb = eo.hfq4_expert_bytes(H, I)
    peak, peak_kind = peaks()
    store = ExpertStore(torch, L, E, H, I, fill_for(torch, synth, W, w))
    dual = DualModel(torch, eo, store, hugepage=args.hugepage)
    pcie = measure_pcie(torch, eo)
    bw_pcie = max(pcie.values())
    counts = W.calibration_counts(w, 1024)
    inp = StackInputs(torch, W, w, L, 1, 16)
    res = {"pcie": pcie}
    for N in w.extra["resident_layers"]:
        for h in w.extra["hot_per_layer"]:
            if N == L and h:
                continue                                  # no host layer to keep hot experts of
            loc, _, hn, hs = eo.hfq_placement_build(counts, eb, N, h, 170 * 2**30)
            layers = dual.layers(loc)
            per_group = [step_bytes(inp.logits[g], k, eb, loc) for g in range(inp.G)]
            timer = StackTimer(torch, eo, layers, inp, k, H, I, E)
            steps = K if N >= 24 else max(5, K // 4)
            total_ms, per_launch, clocks = timer.run(steps, max(3, W_ // 4))
            hbm_b = sum(per_group[i % inp.G][0] for i in range(steps)) / steps
            host_b = sum(per_group[i % inp.G][1] for i in range(steps)) / steps
            roof = offload_roofline(inp.logits, k, eb, loc, hbm_b, host_b, sum(per_launch) / steps,
                                    peak, peak_kind, bw_pcie, pcie, kernel_name(1, 1))
            roof.pop("pcie")
            res[f"offload_n{N}_h{h}"] = sub_result(
                1, steps, total_ms, per_launch, clocks, roof, 1,
                {"workload": w.name, "resident_layers": N, "hot_per_layer": h,
                 "hbm_expert_bytes": hn, "host_expert_bytes": hs,
                 "host_pages": "2 MiB (madvise)" if args.hugepage else "4 KiB"})
            timer.close()
    res.update(run_cache_suite(args, torch, eo, dual, w, K, W_, bw_pcie, peak, peak_kind))
    dual.close()
    # host arena page size (Strata report, pitfall 7): the all-host row again,
    # with the arena on 2 MiB transparent huge pages (madvise, then registered)
    if not args.hugepage:
        before = thp_state()
        dual = DualModel(torch, eo, store, hugepage=True)
        after = thp_state()
        pcie2 = measure_pcie(torch, eo, flags=eo.ARENA_HUGEPAGE)
        loc, _, hn, hs = eo.hfq_placement_build(counts, eb, 0, 0, 170 * 2**30)
        layers = dual.layers(loc)
        per_group = [step_bytes(inp.logits[g], k, eb, loc) for g in range(inp.G)]
        timer = StackTimer(torch, eo, layers, inp, k, H, I, E)
        steps = max(5, K // 4)
        total_ms, per_launch, clocks = timer.run(steps, max(3, W_ // 4))
        hbm_b = sum(per_group[i % inp.G][0] for i in range(steps)) / steps
        host_b = sum(per_group[i % inp.G][1] for i in range(steps)) / steps
        roof = offload_roofline(inp.logits, k, eb, loc, hbm_b, host_b, sum(per_launch) / steps,
                                peak, peak_kind, max(pcie2.values()), pcie2, kernel_name(1, 1))
        roof.pop("pcie")
        res["offload_n0_h0_hugepage"] = sub_result(
            1, steps, total_ms, per_launch, clocks, roof, 1,
            {"workload": w.name, "resident_layers": 0, "hot_per_layer": 0,
             "host_pages": "2 MiB transparent huge pages asked for (madvise)",
             "pcie_hugepage_arena": pcie2, "thp_before": before, "thp_after_arena": after})
        timer.close()
        dual.close()
    store.close()
    del store, dual
    torch.cuda.empty_cache()
    return res


def run_cache_suite(args, torch, eo, dual, w, K, W_, bw_pcie, peak, peak_kind):
    """Every expert of the 48 x 512 model in pinned host memory (N = 0), with
    a dynamic VRAM expert cache in front of it (Strata report, "model and
    engine") and, for comparison, with copy-engine staging of each layer's
    selected experts before the layer runs (the alternative the hipfire
    offload explainer's "PCIe pass-through" section argues against).

    Cache: each step's routing (idx_all) and the location tables the step's
    kernel read are copied to the host behind the kernel; while the next step
    runs, the routing goes to hfq_cache_observe layer by layer, which admits
    up to 4 missed experts per layer (frequency policy) and enqueues their
    copies (copy engine) and table rewrites behind that next step, so they
    serve the step after it.  Misses are read zero-copy meanwhile.  The hit
    rate is counted from the tables each kernel read.  Every step routes a new
    token (skewed routing, 51 hot experts of 512 per layer).  Staging: per
    layer, route on the device, copy the ids to the host, copy the selected
    experts into 8 HBM slots, run the layer."""
    import time

    import numpy as np

    from synth import workloads as W
    L, E, H, I, k = w.layers, w.experts, w.hidden, w.inter, w.top_k
    eb = dual.store.eb
    offs = (np.arange(L * E, dtype=np.uint64) * np.uint64(eb)).reshape(L, E)
    home = offs + np.uint64(dual.host_dev)
    host_src = offs + np.uint64(dual.host)
    home_loc = np.ones((L, E), np.uint8)
    warm, timed = max(64, 8 * W_), max(32, K)
    inp = StackInputs(torch, W, w, L, 1, warm + timed, token0=1 << 20)
    stream = torch.cuda.current_stream()
    ws = torch.zeros(eo.hfq4_stack_workspace_bytes(1, k, H, I, E), dtype=torch.uint8, device="cuda")
    x_out = torch.empty((1, H), dtype=torch.int16, device="cuda")
    wts_all = torch.empty((L, 1, k), dtype=torch.float32, device="cuda")
    idx_dev = [torch.empty((L, 1, k), dtype=torch.int32, device="cuda") for _ in range(2)]
    idx_host = [torch.empty((L, 1, k), dtype=torch.int32).pin_memory() for _ in range(2)]
    loc_host = [torch.empty(L * E, dtype=torch.uint8).pin_memory() for _ in range(2)]
    res = {}
    for slots in (51, 128):
        slot_mem = torch.empty(L * slots * eb, dtype=torch.uint8, device="cuda")
        table = torch.empty(L * E, dtype=torch.int64, device="cuda")
        locd = torch.empty(L * E, dtype=torch.uint8, device="cuda")
        cache = eo.ExpertCache(L, E, eb, slots, home, host_src, home_loc, slot_mem, table, locd, stream)
        layers = [eo.Layer(table[l * E:(l + 1) * E], E, H, I, expert_loc=locd[l * E:(l + 1) * E])
                  for l in range(L)]
        arr = eo.layer_array(layers)
        done = [torch.cuda.Event(), torch.cuda.Event()]
        kev = []
        counts = [0, 0]                                   # hits, selections (distinct per layer)

        def step(g, timed_step):
            b = g & 1
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            eo.hfq4_moe_decode_stack(layers, inp.d_logits[g], k, inp.d_x[g], 1, x_out, ws,
                                     idx_all=idx_dev[b], wts_all=wts_all, _layer_array=arr)
            e1.record()
            idx_host[b].copy_(idx_dev[b], non_blocking=True)
            loc_host[b].copy_(locd, non_blocking=True)    # the tables this kernel read
            done[b].record()
            if timed_step:
                kev.append((e0, e1))
            if g == 0:
                return
            # the previous step's routing, while this step runs
            done[b ^ 1].synchronize()
            ids = idx_host[b ^ 1].numpy().reshape(L, k)
            if timed_step:
                loc = loc_host[b ^ 1].numpy().reshape(L, E)
                for l in range(L):
                    sel = np.unique(ids[l])
                    counts[0] += int((loc[l, sel] == 0).sum())
                    counts[1] += len(sel)
            for l in range(L):
                cache.observe(l, ids[l], 4)

        for g in range(warm):
            step(g, False)
        torch.cuda.synchronize()
        before = cache.stats()
        sampler = ClockSampler(0)
        sampler.start()
        t0 = time.perf_counter()
        for g in range(warm, warm + timed):
            step(g, True)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
        clocks = sampler.stop()
        after = cache.stats()
        eo.hfq_workspace_status(ws)
        kern_ms = [a.elapsed_time(b_) for a, b_ in kev]
        res[f"offload_n0_cache{slots}"] = {
            "value": round(timed / dt, 2), "unit": "tokens/s", "ms_per_step": round(dt / timed * 1e3, 4),
            "steps": timed, "tokens_per_step": 1, "workload": w.name,
            "timing": "host wall clock per step; the cache update of a step (host policy, copy-engine "
                      "refill, table rewrites) overlaps the next step's kernel",
            "cache_slots_per_layer": slots,
            "hit_rate": round(counts[0] / max(1, counts[1]), 4),
            "hit_rate_counted_as": "distinct selected experts per layer that the step's kernel read from HBM",
            "admitted_per_step": round((after["admitted"] - before["admitted"]) / timed, 3),
            "kernel_ms_per_step": round(sum(kern_ms) / len(kern_ms), 4),
            "warmup_steps": warm, "gpu_launches": timed, "clocks": clocks}
        cache.close()
        del slot_mem, table, locd
    # staging before use: per layer route, copy ids to the host, stage, run
    slots = k
    slot_mem = torch.empty(L * slots * eb, dtype=torch.uint8, device="cuda")
    table = torch.empty(L * E, dtype=torch.int64, device="cuda")
    locd = torch.empty(L * E, dtype=torch.uint8, device="cuda")
    cache = eo.ExpertCache(L, E, eb, slots, home, host_src, home_loc, slot_mem, table, locd, stream)
    layers = [eo.Layer(table[l * E:(l + 1) * E], E, H, I, expert_loc=locd[l * E:(l + 1) * E])
              for l in range(L)]
    idx1 = torch.empty((1, k), dtype=torch.int32, device="cuda")
    w1 = torch.empty((1, k), dtype=torch.float32, device="cuda")
    idx1_host = torch.empty((1, k), dtype=torch.int32).pin_memory()
    xa = torch.empty((1, H), dtype=torch.int16, device="cuda")
    xb = torch.empty((1, H), dtype=torch.int16, device="cuda")

    def staged_token(g):
        cur = inp.d_x[g]
        for l in range(L):
            eo.moe_route(inp.d_logits[g, l], 1, E, k, idx1, w1)
            idx1_host.copy_(idx1, non_blocking=True)
            torch.cuda.synchronize()
            cache.observe(l, idx1_host.numpy().ravel(), -1)
            nxt = xa if l % 2 == 0 else xb
            eo.hfq4_moe_decode_stack(layers[l:l + 1], inp.d_logits[g, l], k, cur, 1, nxt, ws)
            cur = nxt
        torch.cuda.synchronize()

    n_staged = max(3, min(8, K // 4))
    for g in range(2):
        staged_token(g)
    t0 = time.perf_counter()
    for g in range(2, 2 + n_staged):
        staged_token(g)
    dt = time.perf_counter() - t0
    eo.hfq_workspace_status(ws)
    res["offload_n0_staged"] = {
        "value": round(n_staged / dt, 2), "unit": "tokens/s", "ms_per_step": round(dt / n_staged * 1e3, 4),
        "steps": n_staged, "tokens_per_step": 1, "workload": w.name,
        "timing": "host wall clock per token: per layer route + idx copy + copy-engine staging of the "
                  "selected experts + the layer",
        "pcie_gbs_measured": bw_pcie, "gpu_launches": 2 * L * n_staged}
    cache.close()
    return res


def run_prefill(args, tokens, K, W_, gemv=True):
    """Prefill chunks through one MoE layer (512 experts, Zipf(1.1) expert
    popularity): a step routes T tokens with grouping by expert (moe_route)
    and runs hfq4_moe_forward, on the tensor-core path (the default for T > 8)
    and, for comparison, on the GEMV path.  Each step routes a different chunk
    of tokens (distinct logits and activations cycled); 256 MB are written
    between timed steps so that the weights come from HBM."""
    import numpy as np
    import torch

    import expert_offload_b200 as eo
    import synth
    from expert_offload_b200.model import ExpertStore
    from synth import workloads as W

    w = W.WORKLOADS[4]
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    eb = eo.hfq4_expert_bytes(H, I)
    store = ExpertStore(torch, 1, E, H, I, fill_for(torch, synth, W, w))
    peak, peak_kind = bf16_peak()
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    res = {}
    for T in tokens:
        G = 2 if T >= 4096 else 4
        logits = torch.from_numpy(np.stack([W.zipf_logits(w, 0, g * T, T) for g in range(G)])).cuda()
        xs = torch.from_numpy(np.stack([W.activations(w, g * T, T)[0] for g in range(G)])
                              .view(np.int16)).cuda()
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
        cnt = torch.empty(E, dtype=torch.int32, device="cuda")
        off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
        rws = torch.zeros(max(256, eo.hfq_route_workspace_bytes(T, E, k)), dtype=torch.uint8,
                          device="cuda")
        y = torch.empty((T, H), dtype=torch.float32, device="cuda")
        ws = torch.zeros(eo.hfq4_moe_workspace_bytes(T, k, H, I, E), dtype=torch.uint8,
                         device="cuda")

        def step(g, path):
            eo.moe_route(logits[g], T, E, k, idx, wts, cnt, off, perm, rws, stream=stream)
            eo.hfq4_moe_forward(store.layers[0], xs[g], eo.HFQ_BF16, T, idx, wts, k, y, ws,
                                cnt=cnt, off=off, perm=perm, path=path, stream=stream)

        def timed(path, steps):
            with torch.cuda.stream(stream):
                for i in range(W_):
                    step(i % G, path)
                torch.cuda.synchronize()
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(steps)]
                for i in range(steps):
                    flush.fill_(i & 0xFF)
                    ev[i][0].record(stream)
                    step(i % G, path)
                    ev[i][1].record(stream)
                torch.cuda.synchronize()
            eo.hfq_workspace_status(ws, stream)
            return sum(a.elapsed_time(b) for a, b in ev) / steps

        sampler = ClockSampler(0)
        sampler.start()
        ms_tc = timed(eo.PATH_AUTO, K)
        clocks = sampler.stop()
        used = int((cnt > 0).sum().item())
        flops = 2.0 * T * k * 3 * H * I
        achieved = flops / (ms_tc / 1e3) / 1e12
        r = {"value": round(T / (ms_tc / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms_tc, 5),
             "steps": K, "tokens_per_step": T, "workload": w.name,
             "path": "tcgen05 grouped dequant-to-bf16 GEMM",
             "experts_used": used, "expert_bytes": used * eb,
             # per step: moe_route (route, group histogram, scan, scatter) and the
             # tensor-core forward (plan, gather, gate/up, down, combine)
             "gpu_launches": (4 + 5) * K, "clocks": clocks,
             "l2": "256 MB written between timed steps",
             "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                          "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                          "flops_per_step": flops, "peak_source": peak_kind,
                          "hbm_time_floor_ms": round(used * eb / (peaks()[0] * 1e9) * 1e3, 4)}}
        if gemv:
            ms_gemv = timed(eo.PATH_GEMV, max(3, min(K, 10)))
            r["gemv_path_ms_per_step"] = round(ms_gemv, 4)
            r["gemv_path_tokens_per_s"] = round(T / (ms_gemv / 1e3), 1)
        res[f"prefill_t{T}"] = r
        del logits, xs, idx, wts, cnt, off, perm, rws, y, ws
    store.close()
    del store, flush
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------- oracle (CPU) arms

def blas_single_threaded():
    """Raises unless every BLAS/OpenMP pool numpy uses has one thread."""
    import numpy  # noqa: F401
    from threadpoolctl import threadpool_info
    pools = threadpool_info()
    bad = [p for p in pools if p.get("num_threads") != 1]
    if bad:
        raise RuntimeError(f"oracle thread pools not limited to one thread: {bad}")
    return len(pools)


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_layer_loop(w, layers, seconds, barrier=None):
    """Runs the oracle on one token through `layers` (cycled) for about
    `seconds`: route, HFQ4 dequantisation of the 8 selected experts and the
    fp64 expert FFNs, residual add.  Packing is load time and not timed.
    Returns (layer passes done, seconds taken)."""
    from oracle import hfq4, moe, route
    from synth import workloads as W

    blas_single_threaded()
    x = W.activations_value(w, 0, 1)
    prep = []
    for l in layers:
        lg = W.logits(w, l, 0, 1)
        idx, _ = route.route(lg, w.top_k)
        ex = {int(e): hfq4.pack_expert(*W.expert_matrices(w, l, int(e))) for e in idx[0]}
        prep.append((lg, ex))
    if barrier is not None:
        barrier.wait()
    n = 0
    t0 = time.perf_counter()
    while True:
        lg, ex = prep[n % len(prep)]
        idx, wts = route.route(lg, w.top_k)
        cache = moe.ExpertCache(ex, w.hidden, w.inter)
        y = moe.moe_layer(cache, w.hidden, w.inter, x, idx, wts)
        x = moe.round_bf16(x + y)
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            return n, dt


def _oracle_worker(args):
    wid, layers, seconds, barrier = args
    from synth import workloads as W
    return _oracle_layer_loop(W.WORKLOADS[2], layers, seconds, barrier)


def cpu_baseline(w, seconds):
    """The oracle as it stands on the host's cores: one core, then one
    process per core (each on its own layers of the stack, all at once).
    tokens/s = layer passes / s / L."""
    import multiprocessing as mp

    n, dt = _oracle_layer_loop(w, [0, 1, 2], seconds)
    one = n / dt / w.layers
    ncpu = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    procs = max(1, min(ncpu, 64))
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    barrier = mgr.Barrier(procs)
    jobs = [(i, [i % w.layers], seconds, barrier) for i in range(procs)]
    with ctx.Pool(procs) as pool:
        outs = pool.map(_oracle_worker, jobs)
    mgr.shutdown()
    allc = sum(n_ / dt_ for n_, dt_ in outs) / w.layers
    return {"value": round(one, 6), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "threads_verified": "BLAS and OpenMP pools at 1 thread (threadpoolctl)",
            "sample": f"1 token through layers 0..2 of the {w.layers}-layer stack, cycled for "
                      f"{dt:.1f} s ({n} layer passes: route, HFQ4 dequantisation of 8 experts, "
                      f"fp64 expert FFNs); tokens/s = passes/s / {w.layers}",
            "all_cores": {"value": round(allc, 6), "unit": "tokens/s", "cores": procs,
                          "nproc": ncpu, "cpu_model": cpu_model(),
                          "sample": f"{procs} independent oracle processes (one per core, "
                                    f"single-threaded each), process i on layer i mod "
                                    f"{w.layers}, {seconds:.0f} s each at once"}}


def run_reference(args):
    """The oracle as the reference arm: each step runs the oracle's HFQ4
    dequantise + fp64 GEMV over a bounded byte sample of one token's work
    (rows of the selected experts of a layer), sized so that the whole run
    stays within a few minutes; tokens/s = bytes/s / bytes per token."""
    from oracle import hfq4, moe, route
    from synth import workloads as W

    blas_single_threaded()
    w = W.WORKLOADS[2]
    H, I, k, L = w.hidden, w.inter, w.top_k, w.layers
    eb = hfq4.expert_bytes(H, I)
    bytes_per_token = L * k * eb
    idx, wts = route.route(W.logits(w, 0, 0, 1), k)
    experts = [hfq4.pack_expert(*W.expert_matrices(w, 0, int(e))) for e in idx[0][:2]]
    x = W.activations_value(w, 0, 1)[0]
    row_bytes = hfq4.matrix_bytes(1, H)
    budget = min(0.5, 150.0 / max(1, args.steps + args.warmup))
    # calibrate rows per step on 64 gate rows
    t0 = time.perf_counter()
    hfq4.dequantize_exact(experts[0][:64 * row_bytes], 64, H) @ x
    per_row = (time.perf_counter() - t0) / 64
    rows = int(max(1, min(I, budget / max(per_row, 1e-9))))

    def one_step(i):
        ex = experts[i % len(experts)]
        r0 = (i * rows) % (I - rows + 1) if rows < I else 0
        g = hfq4.dequantize_exact(ex[r0 * row_bytes:(r0 + rows) * row_bytes], rows, H) @ x
        mg = hfq4.matrix_bytes(I, H)
        u = hfq4.dequantize_exact(ex[mg + r0 * row_bytes:mg + (r0 + rows) * row_bytes], rows, H) @ x
        return moe.silu(g) * u

    for i in range(args.warmup):
        one_step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one_step(i)
    dt = time.perf_counter() - t0
    bytes_done = args.steps * 2 * rows * row_bytes
    value = bytes_done / dt / bytes_per_token
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "layers": L, "hidden": H, "inter": I,
                       "experts": w.experts, "top_k": k, "tokens_per_step": 1},
            "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s", "cores": 1,
                             "kind": "oracle",
                             "sample": f"each step: {rows} gate + {rows} up rows of one selected "
                                       f"expert (HFQ4 dequantise + fp64 GEMV + SiLU*up); "
                                       f"tokens/s = HFQ4 bytes/s / {bytes_per_token} bytes per "
                                       f"token"},
            "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------- main

def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    torch.cuda.set_device(local_rank)
    if args.workload == "routed":
        if rank == 0:
            r = run_routed(args, args.steps, args.warmup)["decode_routed"]
            out = {"metric": METRIC, "n_gpus": 1, "warmup": args.warmup, "higher_is_better": True,
                   "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic"}
            out.update(r)
            out["config"] = {"workload": out.pop("workload")}
            print(json.dumps(out), flush=True)
        return
    if args.workload == "prefill":
        if rank == 0:
            r = run_prefill(args, [args.tokens], args.steps, args.warmup)
            out = {"metric": METRIC, "n_gpus": 1, "warmup": args.warmup, "higher_is_better": True,
                   "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}
            out.update(r[f"prefill_t{args.tokens}"])
            out["config"] = {"workload": out.pop("workload"), "tokens": args.tokens}
            print(json.dumps(out), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    out, w = run_headline(args, rank, world, local_rank, dist)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    if world == 1 and args.workload is None and not args.no_suite:
        # the other configurations, each with fewer steps than the headline
        K = max(5, min(args.steps, 50))
        W_ = max(3, min(args.warmup, 10))
        subs = {}
        subs.update(run_routed(args, K, W_))
        subs.update(run_verify_suite(args, K, W_))
        subs.update(run_offload_suite(args, K, W_))
        subs.update(run_prefill(args, [512, 2048, 8192], K, W_))
        out["workloads"] = subs
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
