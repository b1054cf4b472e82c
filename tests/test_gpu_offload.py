"""GPU parity of the expert-offload path: experts of later layers live in a
pinned, mapped host arena and the same persistent kernel reads them over
PCIe (hipfire offload explainer, "PCIe pass-through"); placement follows the
layer split plus per-layer hot sets ("placement algorithm")."""
import numpy as np
import pytest

import synth
from oracle import moe, placement, route
from synth import workloads as W
from tests.gpu_util import TOL, OraclePackedLayer, device_fill, report

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


@pytest.fixture(scope="module", params=[False, True], ids=["4k_pages", "2m_pages"])
def offload_model(eo, request):
    """Layers 0..2 of the 512-expert model; layer 0 in HBM, layers 1-2 on the
    host except their 51 hottest experts (by calibration counts).  The host
    arena is made both ways: pinned 4 KiB pages (cudaHostAlloc) and 2 MiB
    transparent huge pages asked for with madvise, then registered (the
    Strata report, pitfall 7)."""
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[5]
    L, E = 3, w.experts
    counts = W.calibration_counts(w, 256)[:L]
    eb = eo.hfq4_expert_bytes(w.hidden, w.inter)
    loc, slot, hn, hs = eo.hfq_placement_build(counts, eb, 1, 51, 10 * 2**30)
    ref = placement.place(counts, eb, 1, 51, 10 * 2**30)
    np.testing.assert_array_equal(loc, ref.loc)
    np.testing.assert_array_equal(slot, ref.slot)
    assert int(loc.sum()) == 2 * (E - 51)
    store = ExpertStore(torch, L, E, w.hidden, w.inter, device_fill(torch, w), loc=loc, slot=slot,
                        hugepage=request.param)
    yield w, store, loc
    store.close()


@pytest.mark.parametrize("T", [1, 2, 8])
def test_offloaded_stack_matches_oracle(eo, offload_model, T):
    w, store, loc = offload_model
    H, I, E, k, L = w.hidden, w.inter, w.experts, w.top_k, 3
    logits = np.stack([W.logits(w, l, 300 + T, T) for l in range(L)])
    x0, _ = W.activations(w, 300 + T, T)
    d_logits = torch.from_numpy(logits).cuda()
    d_x0 = torch.from_numpy(x0.view(np.int16)).cuda()
    x_out = torch.empty((T, H), dtype=torch.int16, device="cuda")
    y_all = torch.empty((L, T, H), dtype=torch.float32, device="cuda")
    wsb = torch.zeros(eo.hfq4_stack_workspace_bytes(T, k, H, I, E), dtype=torch.uint8,
                      device="cuda")
    eo.hfq4_moe_decode_stack(store.layers, d_logits, k, d_x0, T, x_out, wsb, y_all=y_all)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(wsb)
    # some selected experts must really come from the host arena
    used_host = sum(int(loc[l, e]) for l in range(L)
                    for e in route.route(logits[l], k)[0].ravel())
    assert used_host > 0
    caches = [moe.ExpertCache(OraclePackedLayer(w, l), H, I) for l in range(L)]
    ys, _ = moe.residual_stack(caches, logits, synth.bf16_bits_to_f32(x0).astype(np.float64), k,
                               route.route)
    errs = [report(y_all.cpu().numpy()[l], ys[l]) for l in range(L)]
    assert max(errs) <= TOL, errs


def test_host_bytes_are_the_packed_experts(eo, offload_model):
    w, store, loc = offload_model
    oracle_l1 = OraclePackedLayer(w, 1)
    host_experts = np.nonzero(loc[1])[0][:3]
    for e in host_experts:
        np.testing.assert_array_equal(store.expert_bytes_at(1, int(e)), oracle_l1[int(e)])


def test_arena_refusal_is_loud(eo):
    counts = np.zeros((48, 512), np.uint32)
    eb = eo.hfq4_expert_bytes(2048, 512)
    with pytest.raises(eo.HfqError) as e:
        eo.hfq_placement_build(counts, eb, 48, 0, 20 * 2**30)
    assert e.value.status == -4 and "deficit" in e.value.message


def test_probe_reads_host_and_device(eo):
    n = 64 << 20
    h, d = eo.hfq_host_arena_create(n)
    try:
        sink = torch.zeros(1, dtype=torch.int64, device="cuda")
        eo.hfq_probe_read(d, n, 1, sink)
        buf = torch.ones(n // 4, dtype=torch.int32, device="cuda")
        eo.hfq_probe_read(buf, n, 2, sink)
        torch.cuda.synchronize()
    finally:
        eo.hfq_host_arena_destroy(h)
