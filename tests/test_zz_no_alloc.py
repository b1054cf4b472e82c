"""The allocation-free forward entry point against the regular one.

hfq4_moe_forward_noalloc serves callers that cannot allocate device memory
(graph-capturing frameworks that own the allocator, allocation-free serving
loops, plugins without an allocator): it keeps its scratch in a fixed device
array inside the library instead of a caller-provided workspace.  Two calls in
a row, on different tokens, must each match hfq4_moe_forward on the same
inputs within the parity tolerance; so must calls that change k from one to
the next, calls with f32 activations, and the call after a bounded wait that
ran out.  This file is collected last so that a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest

import synth
from synth import workloads as W
from tests.gpu_util import TOL, device_fill, report

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def eo():
    assert torch.cuda.is_available()
    synth.build()
    from expert_offload_b200 import build
    build.build()
    import expert_offload_b200
    return expert_offload_b200


@pytest.fixture(scope="module")
def layer6(eo):
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[2]
    store = ExpertStore(torch, 1, w.experts, w.hidden, w.inter,
                        lambda l, g, u, d: device_fill(torch, w)(6, g, u, d))
    return w, store


def _inputs(eo, w, token0, T, k, f32=False):
    logits = torch.from_numpy(W.logits(w, 6, token0, T)).cuda()
    x, _ = W.activations(w, token0, T)
    if f32:
        x = torch.from_numpy(synth.bf16_bits_to_f32(x).astype(np.float32)).cuda()
    else:
        x = torch.from_numpy(x.view(np.int16)).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    eo.moe_route(logits, T, w.experts, k, idx, wts)
    return x, idx, wts


def _reference(eo, layer, x, dtype, T, idx, wts, k, H, I, E):
    """hfq4_moe_forward on a workspace of its own."""
    ws = torch.zeros(eo.hfq4_moe_workspace_bytes(T, k, H, I, E), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.float32, device="cuda")
    eo.hfq4_moe_forward(layer, x, dtype, T, idx, wts, k, y, ws)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(ws)
    return y.cpu().numpy().astype(np.float64)


def _noalloc(eo, layer, x, dtype, T, idx, wts, k, H):
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    eo.hfq4_moe_forward_noalloc(layer, x, dtype, T, idx, wts, k, y)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(None)          # the array's status word: no error
    return y.cpu().numpy()


@pytest.mark.parametrize("T", [1, 5])
def test_noalloc_matches_forward_on_two_calls_in_a_row(eo, layer6, T):
    w, store = layer6
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    layer = store.layers[0]
    for call, token0 in enumerate((900, 1300)):
        x, idx, wts = _inputs(eo, w, token0, T, k)
        ref = _reference(eo, layer, x, eo.HFQ_BF16, T, idx, wts, k, H, I, E)
        got = _noalloc(eo, layer, x, eo.HFQ_BF16, T, idx, wts, k, H)
        assert np.all(np.isfinite(got)), f"call {call}: output not fully written"
        assert report(got, ref) <= TOL, f"call {call}"


def test_noalloc_allocates_no_device_memory(eo, layer6):
    """After a first call on the device (which resolves the array's address),
    a call leaves the device's free memory exactly as it was."""
    w, store = layer6
    H, k = w.hidden, w.top_k
    x, idx, wts = _inputs(eo, w, 77, 1, k)
    y = torch.empty((1, H), dtype=torch.float32, device="cuda")
    eo.hfq4_moe_forward_noalloc(store.layers[0], x, eo.HFQ_BF16, 1, idx, wts, k, y)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        eo.hfq4_moe_forward_noalloc(store.layers[0], x, eo.HFQ_BF16, 1, idx, wts, k, y)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_calls_that_change_k(eo, layer6):
    """A k = 16 call, then 8191 k = 8 calls, then k = 16 again: the last call's
    launch counter is 8192 past the first one's, the one-token kernel's tags
    keep 13 bits of it, and the k = 16 exchange words the k = 8 calls never
    touched still hold the first call's tags.  The layout change must clear
    them, so the last call matches the regular entry point."""
    w, store = layer6
    H, I, E = w.hidden, w.inter, w.experts
    layer = store.layers[0]
    x16, idx16, wts16 = _inputs(eo, w, 2000, 1, 16)
    y16 = torch.empty((1, H), dtype=torch.float32, device="cuda")
    eo.hfq4_moe_forward_noalloc(layer, x16, eo.HFQ_BF16, 1, idx16, wts16, 16, y16)
    x8, idx8, wts8 = _inputs(eo, w, 2100, 1, 8)
    y8 = torch.empty((1, H), dtype=torch.float32, device="cuda")
    for _ in range(8191):
        eo.hfq4_moe_forward_noalloc(layer, x8, eo.HFQ_BF16, 1, idx8, wts8, 8, y8)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(None)
    ref8 = _reference(eo, layer, x8, eo.HFQ_BF16, 1, idx8, wts8, 8, H, I, E)
    assert report(y8.cpu().numpy(), ref8) <= TOL
    x16b, idx16b, wts16b = _inputs(eo, w, 2200, 1, 16)
    got = _noalloc(eo, layer, x16b, eo.HFQ_BF16, 1, idx16b, wts16b, 16, H)
    ref = _reference(eo, layer, x16b, eo.HFQ_BF16, 1, idx16b, wts16b, 16, H, I, E)
    assert report(got, ref) <= TOL


def test_noalloc_f32_activations(eo, layer6):
    """f32 inputs take the general persistent kernel instead of the one-token one."""
    w, store = layer6
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    for T in (1, 3):
        x, idx, wts = _inputs(eo, w, 3000 + T, T, k, f32=True)
        ref = _reference(eo, store.layers[0], x, eo.HFQ_F32, T, idx, wts, k, H, I, E)
        got = _noalloc(eo, store.layers[0], x, eo.HFQ_F32, T, idx, wts, k, H)
        assert report(got, ref) <= TOL, T


def test_noalloc_timeout_is_readable_and_the_next_call_is_correct(eo, layer6):
    """The test hook makes the one-layer launch's h poll expect a tag nobody
    writes: the bounded wait runs out, the array's status word says so through
    hfq_workspace_status(NULL, 0, stream), reading it clears it, and the next
    call is correct."""
    w, store = layer6
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    x, idx, wts = _inputs(eo, w, 4000, 1, k)
    y = torch.empty((1, H), dtype=torch.float32, device="cuda")
    eo.hfq_set_option(eo.OPT_WAIT_TIMEOUT_NS, 20_000_000)
    try:
        eo.hfq_set_option(eo.OPT_TEST_MISSING_ARRIVALS, 1)
        eo.hfq4_moe_forward_noalloc(store.layers[0], x, eo.HFQ_BF16, 1, idx, wts, k, y)
        torch.cuda.synchronize()
        with pytest.raises(eo.HfqError) as e:
            eo.hfq_workspace_status(None)
        assert e.value.status == -6
        eo.hfq_workspace_status(None)
    finally:
        eo.hfq_set_option(eo.OPT_WAIT_TIMEOUT_NS, 1_000_000_000)
    got = _noalloc(eo, store.layers[0], x, eo.HFQ_BF16, 1, idx, wts, k, H)
    ref = _reference(eo, store.layers[0], x, eo.HFQ_BF16, 1, idx, wts, k, H, I, E)
    assert report(got, ref) <= TOL


def test_noalloc_rejects_sizes_beyond_its_scratch(eo):
    lay = eo.Layer(1024, 16, 256, 128)
    lib = eo.lib()
    assert lib.hfq4_moe_forward_noalloc(eo.ctypes.byref(lay.struct), 1024, 0, 9, 1024, 1024, 4,
                                        1024, None, None) == -3
    assert "T <= 8" in eo.last_error()
    wide = eo.Layer(1024, 16, 4096, 128)
    assert lib.hfq4_moe_forward_noalloc(eo.ctypes.byref(wide.struct), 1024, 0, 1, 1024, 1024, 4,
                                        1024, None, None) == -3
    assert "hidden <= 2048" in eo.last_error()
