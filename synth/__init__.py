"""Seeded synthetic inputs for the routed-expert HFQ4 MoE layer.

This module is the one piece that both the oracle side and the CUDA side
consume.  It holds no step of the MoE method (no quantisation, router GEMV,
routing, expert FFN or combine): it only produces the f32 weights,
activations, router weights and logits of the workloads, from counter-based random
numbers (Philox4x32-10, see ``synth_philox.h``) whose bits are identical on
the host (``libsynth_host.so``) and on the GPU (``libsynth_dev.so``).

The pages measure on real models and prompts (a 40-layer MoE with 408 MiB of
experts per layer in the hipfire offload explainer, "placement" and "PCIe
zero-copy" sections); these generators stand in for them with the same
shapes.  The workload recipes are in :mod:`synth.workloads`.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libsynth_host.so")
DEV_SO = os.path.join(HERE, "libsynth_dev.so")

STREAM_WEIGHT = 1
STREAM_ACT = 2
STREAM_LOGIT = 3
STREAM_ROUTER = 4

MAT_GATE, MAT_UP, MAT_DOWN, MAT_ROUTER = 0, 1, 2, 3


def build(verbose: bool = False) -> None:
    """Compile the host (gcc) and device (nvcc, sm_100a) generator libraries."""
    src_h = os.path.join(HERE, "synth_host.c")
    src_d = os.path.join(HERE, "synth_dev.cu")
    hdr = os.path.join(HERE, "synth_philox.h")
    cmds = []
    if _stale(HOST_SO, [src_h, hdr]):
        cmds.append(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-pthread",
                     "-o", HOST_SO, src_h])
    if _stale(DEV_SO, [src_d, hdr]):
        cmds.append(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
                     "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
                     "-fmad=false", "-o", DEV_SO, src_d])
    for c in cmds:
        if verbose:
            print(" ".join(c))
        subprocess.run(c, check=True)


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


_host = None
_dev = None


def host_lib() -> ctypes.CDLL:
    global _host
    if _host is None:
        if not os.path.exists(HOST_SO):
            build()
        lib = ctypes.CDLL(HOST_SO)
        lib.synth_weights_host.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_double, ctypes.c_int]
        lib.synth_weights_host.restype = None
        lib.synth_normal_host.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                          ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int,
                                          ctypes.c_uint64, ctypes.c_double, ctypes.c_int]
        lib.synth_normal_host.restype = None
        lib.synth_normal_fine_host.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                               ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int,
                                               ctypes.c_uint64, ctypes.c_double]
        lib.synth_normal_fine_host.restype = None
        lib.synth_uniform_host.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                           ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64]
        lib.synth_uniform_host.restype = None
        _host = lib
    return _host


def dev_lib() -> ctypes.CDLL:
    global _dev
    if _dev is None:
        if not os.path.exists(DEV_SO):
            raise RuntimeError(f"{DEV_SO} is not built; run synth.build()")
        lib = ctypes.CDLL(DEV_SO)
        lib.synth_weights_dev.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_double, ctypes.c_void_p]
        lib.synth_weights_dev.restype = ctypes.c_int
        lib.synth_normal_dev.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                         ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int,
                                         ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p]
        lib.synth_normal_dev.restype = ctypes.c_int
        _dev = lib
    return _dev


def _threads() -> int:
    return max(1, min(os.cpu_count() or 1, 16))


# ---------------------------------------------------------------- host side

def weights(seed: int, layer: int, expert0: int, n_experts: int, matrix: int, rows: int,
            cols: int, sigma: float, threads: int | None = None) -> np.ndarray:
    """f32 weights [n_experts, rows, cols] of one matrix kind of one layer."""
    out = np.empty((n_experts, rows, cols), dtype=np.float32)
    host_lib().synth_weights_host(out.ctypes.data, seed, layer, expert0, n_experts, matrix,
                                  rows, cols, float(sigma), threads or _threads())
    return out


def normal(seed: int, stream: int, a: int, b0: int, nb: int, per_b: int, sigma: float) -> np.ndarray:
    """f32 samples [nb, per_b] of ~N(0, sigma^2) for tensor (stream, a, b0..b0+nb-1)."""
    out = np.empty((nb, per_b), dtype=np.float32)
    host_lib().synth_normal_host(out.ctypes.data, seed, stream, a, b0, nb, per_b, float(sigma),
                                 _threads())
    return out


def normal_fine(seed: int, stream: int, a: int, b0: int, nb: int, per_b: int,
                sigma: float) -> np.ndarray:
    """f32 [nb, per_b] of ~N(0, sigma^2) with 32-bit resolution (router logits)."""
    out = np.empty((nb, per_b), dtype=np.float32)
    host_lib().synth_normal_fine_host(out.ctypes.data, seed, stream, a, b0, nb, per_b, float(sigma))
    return out


def uniform(seed: int, stream: int, a: int, b: int, n: int) -> np.ndarray:
    """f64 uniforms on (0,1) from 32 random bits each (host-only inputs)."""
    out = np.empty(n, dtype=np.float64)
    host_lib().synth_uniform_host(out.ctypes.data, seed, stream, a, b, n)
    return out


def expert_weights(seed: int, layer: int, expert: int, hidden: int, inter: int,
                   sigma: float = 0.02):
    """(gate [I,H], up [I,H], down [H,I]) f32 weights of one expert."""
    g = weights(seed, layer, expert, 1, MAT_GATE, inter, hidden, sigma)[0]
    u = weights(seed, layer, expert, 1, MAT_UP, inter, hidden, sigma)[0]
    d = weights(seed, layer, expert, 1, MAT_DOWN, hidden, inter, sigma)[0]
    return g, u, d


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round f32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- device side

def weights_dev(out_ptr: int, seed: int, layer: int, expert0: int, n_experts: int, matrix: int,
                rows: int, cols: int, sigma: float, stream: int) -> None:
    rc = dev_lib().synth_weights_dev(out_ptr, seed, layer, expert0, n_experts, matrix, rows, cols,
                                     float(sigma), stream)
    if rc != 0:
        raise RuntimeError(f"synth_weights_dev failed with CUDA error {rc}")


def normal_dev(out_ptr: int, seed: int, stream_id: int, a: int, b0: int, nb: int, per_b: int,
               sigma: float, stream: int) -> None:
    rc = dev_lib().synth_normal_dev(out_ptr, seed, stream_id, a, b0, nb, per_b, float(sigma), stream)
    if rc != 0:
        raise RuntimeError(f"synth_normal_dev failed with CUDA error {rc}")
