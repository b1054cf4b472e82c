"""The allocation-free forward entry point against the regular one.

hfq4_moe_forward_noalloc serves callers that cannot allocate device memory
(graph-capturing frameworks that own the allocator, allocation-free serving
loops, plugins without an allocator): it keeps its scratch in a fixed device
array inside the library instead of a caller-provided workspace.  Two calls in
a row, on different tokens, must each match hfq4_moe_forward on the same
inputs within the parity tolerance.  This file is collected last so that a run
that stops at the first failure has already run every other test."""
import numpy as np
import pytest

import synth
from synth import workloads as W
from tests.gpu_util import TOL, device_fill, max_rel_err

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


@pytest.mark.parametrize("T", [1, 5])
def test_noalloc_matches_forward_on_two_calls_in_a_row(eo, T):
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[2]
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    store = ExpertStore(torch, 1, E, H, I, lambda l, g, u, d: device_fill(torch, w)(6, g, u, d))
    layer = store.layers[0]
    ws = torch.zeros(eo.hfq4_moe_workspace_bytes(T, k, H, I, E), dtype=torch.uint8, device="cuda")
    for call, token0 in enumerate((900, 1300)):
        logits = torch.from_numpy(W.logits(w, 6, token0, T)).cuda()
        x, _ = W.activations(w, token0, T)
        x = torch.from_numpy(x.view(np.int16)).cuda()
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
        eo.moe_route(logits, T, E, k, idx, wts)
        y_ref = torch.empty((T, H), dtype=torch.float32, device="cuda")
        eo.hfq4_moe_forward(layer, x, eo.HFQ_BF16, T, idx, wts, k, y_ref, ws)
        y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
        eo.hfq4_moe_forward_noalloc(layer, x, eo.HFQ_BF16, T, idx, wts, k, y)
        torch.cuda.synchronize()
        ref = y_ref.cpu().numpy().astype(np.float64)
        got = y.cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: output not fully written"
        assert max_rel_err(got, ref) <= TOL, f"call {call}"


def test_noalloc_rejects_sizes_beyond_its_scratch(eo):
    lay = eo.Layer(1024, 16, 256, 128)
    lib = eo.lib()
    assert lib.hfq4_moe_forward_noalloc(eo.ctypes.byref(lay.struct), 1024, 0, 9, 1024, 1024, 4,
                                        1024, None, None) == -3
    assert "T <= 8" in eo.last_error()
