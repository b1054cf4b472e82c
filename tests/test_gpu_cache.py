"""The expert cache on the GPU: the decode stack over cache-managed pointer
tables gives the same bits as over the plain host-mapped tables, while the
copy engine moves experts into HBM slots (refills on the cache's own stream,
named one call later) and the tables switch between a slot and the expert's
host alias (Strata report, "model and engine": a VRAM
cache of hot experts in front of the pinned host arena; hipfire offload
explainer, "PCIe pass-through": the zero-copy reads it competes with)."""
import numpy as np
import pytest

import synth
from oracle import moe, route
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


@pytest.fixture(scope="module")
def host_model(eo):
    """Three layers of the 512-expert model, every expert in the pinned host
    arena (slot = layer * E + expert)."""
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[5]
    L, E = 3, w.experts
    loc = np.ones((L, E), np.uint8)
    slot = np.arange(L * E, dtype=np.int64).reshape(L, E)
    store = ExpertStore(torch, L, E, w.hidden, w.inter, device_fill(torch, w), loc=loc, slot=slot)
    yield w, store
    store.close()


def _stack(eo, layers, logits, x0, k, H, I, E, T=1):
    L = len(layers)
    x_out = torch.empty((T, H), dtype=torch.int16, device="cuda")
    y_all = torch.empty((L, T, H), dtype=torch.float32, device="cuda")
    idx_all = torch.empty((L, T, k), dtype=torch.int32, device="cuda")
    wts_all = torch.empty((L, T, k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(eo.hfq4_stack_workspace_bytes(T, k, H, I, E), dtype=torch.uint8, device="cuda")
    eo.hfq4_moe_decode_stack(layers, logits, k, x0, T, x_out, ws, y_all=y_all, idx_all=idx_all,
                             wts_all=wts_all)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(ws)
    return y_all.cpu().numpy(), idx_all.cpu().numpy()


@pytest.mark.parametrize("max_admit", [4, -1], ids=["refill_between_steps", "stage_before_use"])
def test_cache_managed_tables_give_the_same_bits(eo, host_model, max_admit):
    w, store = host_model
    L, E, H, I, k = 3, w.experts, w.hidden, w.inter, w.top_k
    eb = store.eb
    offs = (np.arange(L * E, dtype=np.uint64) * np.uint64(eb)).reshape(L, E)
    home = offs + np.uint64(store.host_dev)
    host_src = offs + np.uint64(store.host_ptr)
    slots = 16
    slot_mem = torch.empty(L * slots * eb, dtype=torch.uint8, device="cuda")
    table = torch.empty(L * E, dtype=torch.int64, device="cuda")
    locd = torch.empty(L * E, dtype=torch.uint8, device="cuda")
    cache = eo.ExpertCache(L, E, eb, slots, home, host_src, np.ones((L, E), np.uint8), slot_mem,
                           table, locd)
    layers = [eo.Layer(table[l * E:(l + 1) * E], E, H, I, expert_loc=locd[l * E:(l + 1) * E])
              for l in range(L)]
    try:
        for step in range(6):
            token = 700 + step % 3           # tokens come back, so some of their experts hit
            logits = np.stack([W.logits(w, l, token, 1) for l in range(L)])
            x0, _ = W.activations(w, token, 1)
            d_logits = torch.from_numpy(logits).cuda()
            d_x0 = torch.from_numpy(x0.view(np.int16)).cuda()
            if max_admit < 0:
                # staging: the cache holds every selected expert before the launch
                for l in range(L):
                    cache.observe(l, route.route(logits[l], k)[0].ravel(), -1)
                    for e in route.route(logits[l], k)[0].ravel():
                        assert cache.slot_of(l, int(e)) >= 0
            y_c, idx_c = _stack(eo, layers, d_logits, d_x0, k, H, I, E)
            y_z, _ = _stack(eo, store.layers, d_logits, d_x0, k, H, I, E)
            np.testing.assert_array_equal(y_c.view(np.uint32), y_z.view(np.uint32))
            if max_admit >= 0:
                for l in range(L):
                    cache.observe(l, idx_c[l].ravel(), max_admit)
        if max_admit >= 0:
            # refills in flight are named by the flush; the tables then still
            # give the same bits
            cache.flush()
            named = [(l, e) for l in range(L) for e in range(E) if cache.slot_of(l, e) >= 0]
            assert named
            y_c, _ = _stack(eo, layers, d_logits, d_x0, k, H, I, E)
            np.testing.assert_array_equal(y_c.view(np.uint32), y_z.view(np.uint32))
        st = cache.stats()
        assert st["admitted"] > 0 and st["hits"] > 0
        # and the values themselves against the oracle, last token
        caches = [moe.ExpertCache(OraclePackedLayer(w, l), H, I) for l in range(L)]
        ys, _ = moe.residual_stack(caches, logits, synth.bf16_bits_to_f32(x0).astype(np.float64), k,
                                   route.route)
        assert max(report(y_c[l], ys[l]) for l in range(L)) <= TOL
    finally:
        cache.close()
