#!/usr/bin/env python
"""Benchmark of the routed-expert HFQ4 MoE layer on B200.

Default workload: the decode stack of 40 MoE layers (hidden 2048, expert
intermediate 512, 256 experts per layer, top-8, 1 token, bf16 residual
stream), all experts resident in HBM.  A step is one token through all 40
layers: route, gate/up GEMV with SiLU*up, down GEMV with the weighted
combine, residual add.  Every step routes a different token (64 distinct
tokens' logits cycled), so a step streams 535 MB of expert weights, more
than the 126 MB L2: no flush is needed between steps.

Prints one JSON line (rank 0).  --impl reference times the oracle (CPU,
fp64) on bounded samples of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s and achieved GB/s as % of HBM/PCIe roofline"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "verify", "offload", "prefill"], default="decode")
    ap.add_argument("--tokens", type=int, default=8, help="tokens per step (verify, prefill)")
    ap.add_argument("--resident-layers", type=int, default=None, help="offload: N")
    ap.add_argument("--hot", type=int, default=0, help="offload: hot experts per host layer")
    ap.add_argument("--hbm-read-probe", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--distinct-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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


# ------------------------------------------------------------- our arm

def workload_for(args):
    """The workload a run measures (decode by default)."""
    import dataclasses

    from synth import workloads as W
    w = W.WORKLOADS[{"decode": 2, "verify": 3, "offload": 5}[args.workload]]
    if args.layers:
        w = dataclasses.replace(w, layers=args.layers,
                                name=f"{w.name} (first {args.layers} layers)")
    T = args.tokens if args.workload == "verify" else 1
    return w, T


def placement_for(eo, args, w):
    """Location/slot tables: all resident, or the offload split."""
    if args.workload != "offload":
        return None, None, None
    from synth import workloads as W
    counts = W.calibration_counts(w, 1024)
    eb = eo.hfq4_expert_bytes(w.hidden, w.inter)
    N = w.layers if args.resident_layers is None else args.resident_layers
    loc, slot, hn, hs = eo.hfq_placement_build(counts, eb, N, args.hot, 170 * 2**30)
    return loc, slot, {"resident_layers": N, "hot_per_layer": args.hot, "hbm_bytes": hn,
                       "host_bytes": hs}


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


def measure_pcie(torch, eo, nbytes=1 << 30):
    """Host-to-device bandwidth two ways: a pinned cudaMemcpy and the zero-copy
    read kernel over a mapped arena (the strata report's link probe, done here
    with the expert kernel's own load path)."""
    h, d = eo.hfq_host_arena_create(nbytes)
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
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    eo.hfq_probe_read(buf, nbytes, 1, sink)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    eo.hfq_probe_read(buf, nbytes, 3, sink)
    e1.record()
    torch.cuda.synchronize()
    del buf
    return round(3 * nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9, 1)


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


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    import expert_offload_b200 as eo
    import synth
    from expert_offload_b200.model import ExpertStore
    from synth import workloads as W

    w, T = workload_for(args)
    L, H, I, E, k = w.layers, w.hidden, w.inter, w.experts, w.top_k
    eb = eo.hfq4_expert_bytes(H, I)
    G = args.distinct_tokens
    loc, slot, place_info = placement_for(eo, args, w)

    def fill(l, g, u, d):
        s = torch.cuda.current_stream().cuda_stream
        synth.weights_dev(g.data_ptr(), w.seed, l, 0, E, synth.MAT_GATE, I, H, W.WEIGHT_SIGMA, s)
        synth.weights_dev(u.data_ptr(), w.seed, l, 0, E, synth.MAT_UP, I, H, W.WEIGHT_SIGMA, s)
        synth.weights_dev(d.data_ptr(), w.seed, l, 0, E, synth.MAT_DOWN, H, I, W.WEIGHT_SIGMA, s)

    store = ExpertStore(torch, L, E, H, I, fill, loc=loc, slot=slot)
    logits = np.stack([np.stack([W.logits(w, l, g * T, T) for l in range(L)])
                       for g in range(G)])                                       # [G, L, T, E]
    xs = np.stack([W.activations(w, g * T, T)[0] for g in range(G)])            # [G, T, H] bf16
    per_group = [step_bytes(logits[g], k, eb, loc) for g in range(G)]
    d_logits = torch.from_numpy(logits).cuda()
    d_x = torch.from_numpy(xs.view(np.int16)).cuda()
    x_out = torch.empty((G, T, H), dtype=torch.int16, device="cuda")
    ws = torch.zeros(eo.hfq4_stack_workspace_bytes(T, k, H, I, E), dtype=torch.uint8,
                     device="cuda")
    arr = eo.layer_array(store.layers)
    stream = torch.cuda.Stream()

    def step(g, s=None):
        eo.hfq4_moe_decode_stack(store.layers, d_logits[g], k, d_x[g], T, x_out[g], ws,
                                 path=args.path, stream=s, _layer_array=arr)

    with torch.cuda.stream(stream):
        for g in range(G):
            step(g, stream)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(ws, stream)
    graphs = []
    try:
        for g in range(G):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                step(g, stream)
            graphs.append(gr)
        torch.cuda.synchronize()
        replay = [gr.replay for gr in graphs]
        launch_mode = "cuda graph per token group"
    except RuntimeError as exc:          # capture not possible: launch directly
        print(f"graph capture failed ({exc}); launching directly", file=sys.stderr)
        torch.cuda.synchronize()
        graphs = []
        replay = [(lambda g=g: step(g, stream)) for g in range(G)]
        launch_mode = "direct launch"
    launches_per_step = eo.hfq4_stack_launches(L, T, k, H, I)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            replay[i % G]()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    sampler = ClockSampler(local_rank)
    sampler.start()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for i in range(K):
            replay[i % G]()
            ev[i + 1].record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = ev[0].elapsed_time(ev[K])
    per_launch = [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
    eo.hfq_workspace_status(ws, stream)

    # end to end through the C ABI: pinned host inputs copied in, result copied out
    K2 = min(args.e2e_steps, K)
    h_logits = torch.from_numpy(logits).pin_memory()
    h_x = torch.from_numpy(xs.view(np.int16)).pin_memory()
    h_out = torch.empty((G, T, H), dtype=torch.int16).pin_memory()
    in_l = torch.empty_like(d_logits[0])
    in_x = torch.empty_like(d_x[0])
    out_x = torch.empty_like(x_out[0])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_step(i):
        g = i % G
        in_l.copy_(h_logits[g], non_blocking=True)
        in_x.copy_(h_x[g], non_blocking=True)
        eo.hfq4_moe_decode_stack(store.layers, in_l, k, in_x, T, out_x, ws, path=args.path,
                                 stream=stream, _layer_array=arr)
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
    eo.hfq_workspace_status(ws, stream)

    total_ms, e2e_ms = max_over_ranks(dist, [total_ms, e2e_ms], "cuda")

    hbm_b = sum(per_group[i % G][0] for i in range(K)) / K
    host_b = sum(per_group[i % G][1] for i in range(K)) / K
    bytes_per_step = hbm_b + host_b
    value = job_rate(world, K, T, total_ms)
    mean_launch_ms = sum(per_launch) / K
    peak, peak_kind = peaks()
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "layers": L, "hidden": H, "inter": I, "experts": E,
                   "top_k": k, "tokens_per_step": T, "weights": "hfq4 (136-byte blocks)",
                   "activations": "bf16", "accumulate": "f32",
                   "distinct_token_groups_cycled": G,
                   "expert_bytes_per_step": round(bytes_per_step),
                   "launch": launch_mode,
                   "l2": "per-step working set > 126 MB L2 (every step routes new tokens); "
                         "no flush",
                   "parallelism": f"replicas x{world}"},
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    kernel = (("decode1_kernel" if T == 1 else "verify_kernel") +
              " (persistent: all layers of one step per launch)"
              if launches_per_step == 1 else "per-layer route + gate/up + down launches")
    if args.workload == "offload":
        pcie = measure_pcie(torch, eo)
        bw_pcie = max(pcie.values())
        roof_ms = 0.0
        for g in range(G):
            # per layer the HBM and PCIe streams overlap: max of the two, summed
            lg = logits[g]
            for l in range(L):
                hb, hs = step_bytes(lg[l:l + 1], k, eb, loc[l:l + 1])
                roof_ms += max(hb / (peak * 1e9), hs / (bw_pcie * 1e9)) * 1e3
        roof_ms /= G
        out["config"]["placement"] = place_info
        out["config"]["pcie"] = pcie
        out["roofline"] = {"bound": "pcie" if host_b > 0 else "hbm",
                           "achieved": round(bytes_per_step / (mean_launch_ms / 1e3) / 1e9, 2),
                           "peak": round(bytes_per_step / (roof_ms / 1e3) / 1e9, 2),
                           "unit": "GB/s", "frac": round(roof_ms / mean_launch_ms, 4),
                           "traffic": None, "kernel": kernel,
                           "peak_source": f"roofline time from measured PCIe {bw_pcie} GB/s "
                                          f"and {peak_kind} HBM {peak} GB/s per layer",
                           "hbm_bytes_per_launch": round(hbm_b),
                           "host_bytes_per_launch": round(host_b),
                           "mean_launch_ms": round(mean_launch_ms, 5)}
    else:
        achieved = bytes_per_step / (mean_launch_ms / 1e3) / 1e9
        # DRAM bytes (read + write) of decode1_kernel from an ncu capture of the
        # first 10 layers of this workload (133.86 MB read + 4.39 MB written),
        # scaled by 4 to the 40-layer launch (the per-layer work is the same)
        traffic = (133.859072e6 + 4.390912e6) * 4 if (args.workload == "decode" and T == 1
                                                 and L == 40 and not args.layers) else None
        out["roofline"] = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                           "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                           "traffic_unit": "DRAM bytes per launch",
                           "peak_source": peak_kind, "kernel": kernel,
                           "bytes_per_launch": round(bytes_per_step),
                           "mean_launch_ms": round(mean_launch_ms, 5)}
        if args.hbm_read_probe:
            out["roofline"]["hbm_read_probe_gbs"] = measure_hbm_read(torch, eo)
    out["e2e"] = {"value": round(job_rate(world, K2, T, e2e_ms), 2), "unit": "tokens/s",
                  "h2d_bytes_per_step": int(in_l.numel() * 4 + in_x.numel() * 2),
                  "d2h_bytes_per_step": int(out_x.numel() * 2)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    if dist:
        dist.barrier()
        graphs.clear()
        dist.destroy_process_group()
    store.close()
    return out


# ------------------------------------------------------------- prefill arm

def run_prefill(args):
    """One prefill chunk through one MoE layer (512 experts, Zipf(1.1) expert
    popularity): a step routes T tokens with grouping by expert (moe_route)
    and runs hfq4_moe_forward, on the tensor-core path (the default for
    T > 8) and, for comparison, on the GEMV path.  Each step routes a
    different chunk of tokens (distinct logits and activations cycled)."""
    import numpy as np
    import torch

    import expert_offload_b200 as eo
    import synth
    from expert_offload_b200.model import ExpertStore
    from synth import workloads as W

    torch.cuda.set_device(0)
    w = W.WORKLOADS[4]
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, args.tokens
    G = max(2, min(args.distinct_tokens, 8))

    def fill(l, g, u, d):
        s = torch.cuda.current_stream().cuda_stream
        synth.weights_dev(g.data_ptr(), w.seed, l, 0, E, synth.MAT_GATE, I, H, W.WEIGHT_SIGMA, s)
        synth.weights_dev(u.data_ptr(), w.seed, l, 0, E, synth.MAT_UP, I, H, W.WEIGHT_SIGMA, s)
        synth.weights_dev(d.data_ptr(), w.seed, l, 0, E, synth.MAT_DOWN, H, I, W.WEIGHT_SIGMA, s)

    store = ExpertStore(torch, 1, E, H, I, fill)
    logits = torch.from_numpy(np.stack([W.zipf_logits(w, 0, g * T, T) for g in range(G)])).cuda()
    xs = torch.from_numpy(np.stack([W.activations(w, g * T, T)[0] for g in range(G)]).view(np.int16)).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    rws = torch.zeros(max(256, eo.hfq_route_workspace_bytes(T, E, k)), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.float32, device="cuda")
    need = eo.hfq4_moe_workspace_bytes(T, k, H, I, E)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    # 256 MB written between steps flushes the 126 MB L2 (weights of a chunk are < 1 GB)
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def step(g, path):
        eo.moe_route(logits[g], T, E, k, idx, wts, cnt, off, perm, rws, stream=stream)
        eo.hfq4_moe_forward(store.layers[0], xs[g], eo.HFQ_BF16, T, idx, wts, k, y, ws, cnt=cnt,
                            off=off, perm=perm, path=path, stream=stream)

    def timed(path, steps):
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
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
    ms_tc = timed(eo.PATH_AUTO, args.steps)
    clocks = sampler.stop()
    ms_gemv = timed(eo.PATH_GEMV, max(3, min(args.steps, 20)))
    used = int((cnt > 0).sum().item())
    eb = eo.hfq4_expert_bytes(H, I)
    flops = 2.0 * T * k * 3 * H * I
    d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {"bf16_tflops": 1590.0}
    peak = float(d["bf16_tflops"])
    achieved = flops / (ms_tc / 1e3) / 1e12
    out = {"metric": METRIC, "value": round(T / (ms_tc / 1e3), 1), "unit": "tokens/s", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_tc, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic",
           "config": {"workload": w.name, "tokens": T, "layers": 1, "hidden": H, "inter": I,
                      "experts": E, "top_k": k, "path": "tcgen05 grouped dequant-to-bf16 GEMM",
                      "experts_used": used, "expert_bytes": used * eb,
                      "l2": "256 MB written between timed steps",
                      "gemv_path_ms_per_step": round(ms_gemv, 4),
                      "gemv_path_tokens_per_s": round(T / (ms_gemv / 1e3), 1)},
           # per step: moe_route (route, group histogram, scan, scatter) and the
           # tensor-core forward (plan, gather, gate/up, down, combine)
           "gpu_launches": (4 + 5) * args.steps, "clocks": clocks,
           "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                        "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                        "flops_per_step": flops,
                        "hbm_time_floor_ms": round(used * eb / 6522.1e9 * 1e3, 4),
                        "peak_source": "measured bf16 burst"}}
    store.close()
    return out


# ------------------------------------------------------- oracle (CPU) arms

def _threads_one():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(1)
    except ImportError:
        return None


def cpu_baseline(w, layers_sampled: int = 3):
    """The oracle as it stands, single-threaded, on one token through the
    first `layers_sampled` layers of the stack (dequantise the selected
    experts' HFQ4 bytes and run them in fp64); packing is load time and is
    not timed.  tokens/s = 1 / (time per layer x L)."""
    import numpy as np

    from oracle import hfq4, moe, route
    from synth import workloads as W

    lim = _threads_one()
    x = W.activations_value(w, 0, 1)
    packed, routes = [], []
    for l in range(layers_sampled):
        lg = W.logits(w, l, 0, 1)
        idx, wts = route.route(lg, w.top_k)
        ex = {int(e): hfq4.pack_expert(*W.expert_matrices(w, l, int(e))) for e in idx[0]}
        packed.append(ex)
        routes.append((lg, idx, wts))
    t0 = time.perf_counter()
    for l in range(layers_sampled):
        idx, wts = route.route(routes[l][0], w.top_k)
        cache = moe.ExpertCache(packed[l], w.hidden, w.inter)
        y = moe.moe_layer(cache, w.hidden, w.inter, x, idx, wts)
        x = moe.round_bf16(x + y)
    dt = time.perf_counter() - t0
    if lim is not None:
        lim.unregister() if hasattr(lim, "unregister") else None
    return {"value": round(layers_sampled / (dt * w.layers), 6), "unit": "tokens/s", "cores": 1,
            "kind": "oracle",
            "sample": f"1 token through layers 0..{layers_sampled - 1} of the {w.layers}-layer "
                      f"stack ({layers_sampled * w.top_k} expert FFNs, HFQ4 dequantise + fp64 "
                      f"GEMVs), {dt:.1f} s, scaled by {w.layers}/{layers_sampled}"}


def run_reference(args):
    """The oracle as the reference arm: each step runs the oracle's HFQ4
    dequantise + fp64 GEMV over a bounded byte sample of one token's work
    (rows of the selected experts of a layer), sized so that the whole run
    stays within a few minutes; tokens/s = bytes/s / bytes per token."""
    import numpy as np

    from oracle import hfq4, moe, route
    from synth import workloads as W

    lim = _threads_one()
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


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if "WORLD_SIZE" not in os.environ:
        world = 1
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return
    if args.workload == "prefill":
        if rank == 0:
            print(json.dumps(run_prefill(args)), flush=True)
        return
    out = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
