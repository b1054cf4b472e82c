"""Python binding of libhfq4moe.so: the routed-expert HFQ4 MoE layer on B200.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Functions carry the C ABI's names (see include/hfq4moe.h) and take
torch tensors, numpy arrays, raw integer addresses or None for pointers, and
a torch stream, a raw cudaStream_t integer or None (= torch's current stream)
for streams.  A failed call raises HfqError with the library's message.

The library must be built (``python -m expert_offload_b200.build``); there is
no fallback of any kind when it is missing.
"""
from __future__ import annotations

import ctypes
import os
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libhfq4moe.so")

HFQ_OK = 0
STATUS = {0: "HFQ_OK", -1: "HFQ_ERR_ARG", -2: "HFQ_ERR_ALIGN", -3: "HFQ_ERR_UNSUPPORTED",
          -4: "HFQ_ERR_NOFIT", -5: "HFQ_ERR_CUDA", -6: "HFQ_ERR_TIMEOUT", -7: "HFQ_ERR_ALLOC",
          -8: "HFQ_ERR_WORKSPACE"}
HFQ_F32, HFQ_BF16 = 0, 1
PATH_AUTO, PATH_GEMV, PATH_TC = 0, 1, 2
ARENA_HUGEPAGE = 1
BLOCK, BLOCK_BYTES = 256, 136
MAX_EXPERTS, MAX_TOPK, MAX_STACK_LAYERS = 512, 16, 64


class HfqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.message = message


class hfq4_layer(ctypes.Structure):
    _fields_ = [("expert_ptr", ctypes.c_void_p), ("expert_loc", ctypes.c_void_p),
                ("n_experts", ctypes.c_int), ("hidden", ctypes.c_int), ("inter", ctypes.c_int)]


_vp, _i, _sz, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64

# name -> (restype, argtypes)
_SIGS = {
    "hfq_last_error": (ctypes.c_char_p, []),
    "hfq_version": (_i, []),
    "hfq4_matrix_bytes": (_sz, [_i, _i]),
    "hfq4_expert_bytes": (_sz, [_i, _i]),
    "hfq4_pack_experts": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _sz]),
    "hfq4_pack_experts_device": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "hfq4_dequant": (_i, [_vp, _i, _i, _vp, _vp]),
    "hfq_route_workspace_bytes": (_sz, [_i, _i, _i]),
    "moe_route": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "hfq4_moe_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "hfq4_moe_forward": (_i, [ctypes.POINTER(hfq4_layer), _vp, _i, _i, _vp, _vp, _i, _vp, _vp,
                              _vp, _vp, _vp, _i, _vp, _sz, _vp]),
    "hfq4_moe_forward_noalloc": (_i, [ctypes.POINTER(hfq4_layer), _vp, _i, _i, _vp, _vp, _i,
                                      _vp, _vp, _vp]),
    "hfq4_stack_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "hfq4_stack_launches": (_i, [_i, _i, _i, _i, _i]),
    "hfq4_moe_decode_stack": (_i, [ctypes.POINTER(hfq4_layer), _i, _vp, _i, _vp, _i, _vp, _vp,
                                   _vp, _vp, _i, _vp, _sz, _vp]),
    "moe_router_logits": (_i, [_vp, _i, _i, _i, _vp, _i, _i, _vp, _vp]),
    "hfq4_moe_decode_stack_routed": (_i, [ctypes.POINTER(hfq4_layer), _i, _vp, _i, _i, _vp, _i,
                                          _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "hfq_workspace_status": (_i, [_vp, _sz, _vp]),
    "hfq_set_option": (_i, [_i, ctypes.c_longlong]),
    "hfq_host_arena_create": (_i, [_sz, _i, ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    "hfq_host_arena_destroy": (_i, [_vp]),
    "hfq_placement_build": (_i, [_i, _i, _sz, _vp, _i, _i, _sz, _vp, _vp,
                                 ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "hfq_placement_pointers": (_i, [_i, _i, _sz, _vp, _vp, _vp, _vp, _vp]),
    "hfq_probe_read": (_i, [_vp, _sz, _i, _vp, _vp]),
    "hfq_cache_create": (_i, [_i, _i, _sz, _i, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp,
                              ctypes.POINTER(_vp)]),
    "hfq_cache_observe": (_i, [_vp, _i, _vp, _i, _i, _vp]),
    "hfq_cache_flush": (_i, [_vp, _vp]),
    "hfq_cache_slot_of": (_i, [_vp, _i, _i, ctypes.POINTER(_i)]),
    "hfq_cache_stats": (_i, [_vp, ctypes.POINTER(_u64), ctypes.POINTER(_u64), ctypes.POINTER(_u64),
                             ctypes.POINTER(_u64)]),
    "hfq_cache_destroy": (_i, [_vp]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m expert_offload_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype, f.argtypes = res, args
        _lib = l
    return _lib


def symbols():
    """Names of the C entry points this binding declares."""
    return list(_SIGS)


def last_error() -> str:
    return lib().hfq_last_error().decode()


def _check(status: int) -> None:
    if status != HFQ_OK:
        raise HfqError(status, last_error())


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if hasattr(a, "ctypes"):
        return a.ctypes.data
    raise TypeError(f"cannot take the address of {type(a)}")


def _nbytes(a) -> int:
    if hasattr(a, "nbytes") and not callable(a.nbytes):
        return int(a.nbytes)
    return int(a.numel() * a.element_size())


def _stream(s):
    if s is None:
        torch = sys.modules.get("torch")
        if torch is not None and torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ------------------------------------------------------------------ sizes

def hfq4_matrix_bytes(rows: int, cols: int) -> int:
    return lib().hfq4_matrix_bytes(rows, cols)


def hfq4_expert_bytes(hidden: int, inter: int) -> int:
    return lib().hfq4_expert_bytes(hidden, inter)


# ---------------------------------------------------------------- packing

def hfq4_pack_experts(gate, up, down, out, n_experts: int, hidden: int, inter: int) -> None:
    """Host packer: numpy f32 gate/up [E,I,H], down [E,H,I] -> out uint8 bytes."""
    _check(lib().hfq4_pack_experts(_ptr(gate), _ptr(up), _ptr(down), n_experts, hidden, inter,
                                   _ptr(out), _nbytes(out)))


def hfq4_pack_experts_device(gate, up, down, out, n_experts: int, hidden: int, inter: int,
                             stream=None) -> None:
    _check(lib().hfq4_pack_experts_device(_ptr(gate), _ptr(up), _ptr(down), n_experts, hidden,
                                          inter, _ptr(out), _nbytes(out), _stream(stream)))


def hfq4_dequant(blocks, rows: int, cols: int, out, stream=None) -> None:
    _check(lib().hfq4_dequant(_ptr(blocks), rows, cols, _ptr(out), _stream(stream)))


# ------------------------------------------------------------------ route

def hfq_route_workspace_bytes(T: int, E: int, k: int) -> int:
    return lib().hfq_route_workspace_bytes(T, E, k)


def moe_route(logits, T: int, E: int, k: int, idx, wts, cnt=None, off=None, perm=None,
              workspace=None, stream=None) -> None:
    ws_bytes = _nbytes(workspace) if workspace is not None else 0
    _check(lib().moe_route(_ptr(logits), T, E, k, _ptr(idx), _ptr(wts), _ptr(cnt), _ptr(off),
                           _ptr(perm), _ptr(workspace), ws_bytes, _stream(stream)))


def moe_router_logits(x, x_dtype: int, T: int, hidden: int, router, router_dtype: int,
                      n_experts: int, logits, stream=None) -> None:
    """logits [T, E] f32 = x Wr^T on the device."""
    _check(lib().moe_router_logits(_ptr(x), x_dtype, T, hidden, _ptr(router), router_dtype,
                                   n_experts, _ptr(logits), _stream(stream)))


# ---------------------------------------------------------------- forward

class Layer:
    """Keeps an hfq4_layer struct and the device tensors it points to alive."""

    def __init__(self, expert_ptr, n_experts: int, hidden: int, inter: int, expert_loc=None):
        self.expert_ptr, self.expert_loc = expert_ptr, expert_loc
        self.struct = hfq4_layer(_ptr(expert_ptr), _ptr(expert_loc), n_experts, hidden, inter)


def hfq4_moe_workspace_bytes(T: int, k: int, hidden: int, inter: int, n_experts: int) -> int:
    return lib().hfq4_moe_workspace_bytes(T, k, hidden, inter, n_experts)


def hfq4_moe_forward(layer: Layer, x, x_dtype: int, T: int, idx, wts, k: int, y, workspace,
                     y_bf16=None, cnt=None, off=None, perm=None, path: int = PATH_AUTO,
                     stream=None) -> None:
    _check(lib().hfq4_moe_forward(ctypes.byref(layer.struct), _ptr(x), x_dtype, T, _ptr(idx),
                                  _ptr(wts), k, _ptr(cnt), _ptr(off), _ptr(perm), _ptr(y),
                                  _ptr(y_bf16), path, _ptr(workspace), _nbytes(workspace),
                                  _stream(stream)))


def hfq4_moe_forward_noalloc(layer: Layer, x, x_dtype: int, T: int, idx, wts, k: int, y,
                             y_bf16=None, stream=None) -> None:
    """hfq4_moe_forward without a workspace: for callers that cannot allocate
    device memory (scratch is a fixed array inside the library)."""
    _check(lib().hfq4_moe_forward_noalloc(ctypes.byref(layer.struct), _ptr(x), x_dtype, T,
                                          _ptr(idx), _ptr(wts), k, _ptr(y), _ptr(y_bf16),
                                          _stream(stream)))


def hfq4_stack_workspace_bytes(T: int, k: int, hidden: int, inter: int, n_experts: int) -> int:
    return lib().hfq4_stack_workspace_bytes(T, k, hidden, inter, n_experts)


def hfq4_stack_launches(n_layers: int, T: int, k: int, hidden: int, inter: int) -> int:
    return lib().hfq4_stack_launches(n_layers, T, k, hidden, inter)


def layer_array(layers):
    arr = (hfq4_layer * len(layers))()
    for i, l in enumerate(layers):
        arr[i] = l.struct
    return arr


def hfq4_moe_decode_stack(layers, logits, k: int, x0, T: int, x_out, workspace, y_all=None,
                          idx_all=None, wts_all=None, path: int = PATH_AUTO, stream=None,
                          _layer_array=None) -> None:
    arr = _layer_array if _layer_array is not None else layer_array(layers)
    _check(lib().hfq4_moe_decode_stack(arr, len(layers), _ptr(logits), k, _ptr(x0), T, _ptr(x_out),
                                       _ptr(y_all), _ptr(idx_all), _ptr(wts_all), path,
                                       _ptr(workspace), _nbytes(workspace), _stream(stream)))


def hfq4_moe_decode_stack_routed(layers, router, router_dtype: int, k: int, x0, T: int, x_out,
                                 workspace, y_all=None, idx_all=None, wts_all=None,
                                 logits_all=None, stream=None, _layer_array=None) -> None:
    arr = _layer_array if _layer_array is not None else layer_array(layers)
    _check(lib().hfq4_moe_decode_stack_routed(arr, len(layers), _ptr(router), router_dtype, k,
                                              _ptr(x0), T, _ptr(x_out), _ptr(y_all),
                                              _ptr(idx_all), _ptr(wts_all), _ptr(logits_all),
                                              _ptr(workspace), _nbytes(workspace),
                                              _stream(stream)))


OPT_WAIT_TIMEOUT_NS, OPT_TEST_MISSING_ARRIVALS, OPT_TIMELINE_BUFFER = 1, 2, 3


def hfq_set_option(option: int, value: int) -> None:
    _check(lib().hfq_set_option(option, value))


def hfq_workspace_status(workspace, stream=None) -> None:
    """Raises HfqError for a device-side error recorded in the workspace; None
    reads the array of hfq4_moe_forward_noalloc on the current device."""
    nbytes = 0 if workspace is None else _nbytes(workspace)
    _check(lib().hfq_workspace_status(_ptr(workspace), nbytes, _stream(stream)))


# --------------------------------------------------------- offload plumbing

def hfq_host_arena_create(nbytes: int, flags: int = 0):
    """Returns (host_address, device_address) of a pinned, mapped arena."""
    h, d = ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib().hfq_host_arena_create(nbytes, flags, ctypes.byref(h), ctypes.byref(d)))
    return h.value, d.value


def hfq_host_arena_destroy(host: int) -> None:
    _check(lib().hfq_host_arena_destroy(host))


def hfq_placement_build(counts, expert_bytes: int, resident_layers: int, hot_per_layer: int,
                        hbm_budget: int):
    """Returns (loc uint8 [L,E], slot int64 [L,E], hbm_needed, host_needed)."""
    import numpy as np
    counts = np.ascontiguousarray(counts, dtype=np.uint32)
    L, E = counts.shape
    loc = np.zeros((L, E), dtype=np.uint8)
    slot = np.zeros((L, E), dtype=np.int64)
    hn, hs = ctypes.c_size_t(), ctypes.c_size_t()
    st = lib().hfq_placement_build(L, E, expert_bytes, counts.ctypes.data, resident_layers,
                                   hot_per_layer, hbm_budget, loc.ctypes.data, slot.ctypes.data,
                                   ctypes.byref(hn), ctypes.byref(hs))
    if st != HFQ_OK:
        err = HfqError(st, last_error())
        err.hbm_needed, err.host_needed = hn.value, hs.value
        raise err
    return loc, slot, hn.value, hs.value


def hfq_placement_pointers(loc, slot, expert_bytes: int, hbm_base: int, host_dev_base: int):
    import numpy as np
    L, E = loc.shape
    out = np.zeros((L, E), dtype=np.uint64)
    _check(lib().hfq_placement_pointers(L, E, expert_bytes, _ptr(np.ascontiguousarray(loc)),
                                        _ptr(np.ascontiguousarray(slot)), hbm_base, host_dev_base,
                                        out.ctypes.data))
    return out


def hfq_probe_read(src, nbytes: int, iters: int, sink, stream=None) -> None:
    _check(lib().hfq_probe_read(_ptr(src), nbytes, iters, _ptr(sink), _stream(stream)))


# ------------------------------------------------------------ expert cache

class ExpertCache:
    """hfq_cache_* over the pointer (and location) tables of L layers.

    home, host_src: uint64 [L, E] numpy arrays (see include/hfq4moe.h);
    home_loc: uint8 [L, E]; slot_mem, table_dev, loc_dev: device tensors or
    None (table_dev None: bookkeeping only)."""

    def __init__(self, L: int, E: int, expert_bytes: int, slots: int, home, host_src, home_loc,
                 slot_mem=None, table_dev=None, loc_dev=None, stream=None):
        import numpy as np
        self._keep = [np.ascontiguousarray(home, np.uint64), np.ascontiguousarray(host_src, np.uint64),
                      np.ascontiguousarray(home_loc, np.uint8)]
        h = ctypes.c_void_p()
        _check(lib().hfq_cache_create(L, E, expert_bytes, slots, self._keep[0].ctypes.data,
                                      self._keep[1].ctypes.data, self._keep[2].ctypes.data,
                                      _ptr(slot_mem), _nbytes(slot_mem) if slot_mem is not None else 0,
                                      _ptr(table_dev), _ptr(loc_dev), _stream(stream), ctypes.byref(h)))
        self.handle = h.value

    def observe(self, layer: int, ids, max_admit: int, stream=None) -> None:
        import numpy as np
        a = np.ascontiguousarray(ids, np.int32).ravel()
        _check(lib().hfq_cache_observe(self.handle, layer, a.ctypes.data, a.size, max_admit,
                                       _stream(stream)))

    def flush(self, stream=None) -> None:
        """Names the slots of the refills still in flight."""
        _check(lib().hfq_cache_flush(self.handle, _stream(stream)))

    def slot_of(self, layer: int, expert: int) -> int:
        s = ctypes.c_int()
        _check(lib().hfq_cache_slot_of(self.handle, layer, expert, ctypes.byref(s)))
        return s.value

    def stats(self):
        v = [ctypes.c_uint64() for _ in range(4)]
        _check(lib().hfq_cache_stats(self.handle, *[ctypes.byref(x) for x in v]))
        return dict(zip(("hits", "misses", "admitted", "evicted"), (x.value for x in v)))

    def close(self) -> None:
        if self.handle:
            _check(lib().hfq_cache_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except (HfqError, AttributeError, TypeError):
            pass
