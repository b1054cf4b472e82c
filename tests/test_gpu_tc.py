"""GPU parity of the tensor-core (tcgen05) expert path for prefill chunks.

The path computes the same layer with bf16 operands: weights RN_bf16 of their
correctly rounded f32 values, bf16 activations, f32 accumulation, h kept
to about 16 significant bits (two bf16 parts) before the down projection.
The oracle's bf16 model (moe.ExpertCache with tc=True: weights rounded to
bf16, h unrounded) states that; y must match it within 1e-3."""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import moe, route
from synth import workloads as W
from tests.gpu_util import TOL, OraclePackedLayer, device_fill, oracle_rows, report

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


def _route(eo, logits, k):
    T, E = logits.shape
    lg = torch.from_numpy(np.ascontiguousarray(logits)).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    rws = torch.zeros(max(256, eo.hfq_route_workspace_bytes(T, E, k)), dtype=torch.uint8,
                      device="cuda")
    eo.moe_route(lg, T, E, k, idx, wts, cnt, off, perm, rws)
    return idx, wts, cnt, off, perm


def _forward(eo, layer, x_bits, T, k, routed, path, H, I, E):
    idx, wts, cnt, off, perm = routed
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    need = eo.hfq4_moe_workspace_bytes(T, k, H, I, E) * (2 if path == eo.PATH_TC and T <= 8 else 1)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    eo.hfq4_moe_forward(layer, torch.from_numpy(x_bits.view(np.int16)).cuda(), eo.HFQ_BF16, T, idx,
                        wts, k, y, ws, cnt=cnt, off=off, perm=perm, path=path)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(ws)
    return y.cpu().numpy()


@pytest.fixture(scope="module")
def small_layer(eo):
    """32 experts at full H = 2048, I = 512, Zipf(1.1) routing so that the head
    experts span several 128-token tiles."""
    from expert_offload_b200.model import ExpertStore
    w = dataclasses.replace(W.WORKLOADS[4], experts=32)
    store = ExpertStore(torch, 1, 32, w.hidden, w.inter, device_fill(torch, w))
    return w, store


def test_tc_path_all_tokens(eo, small_layer):
    w, store = small_layer
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 256
    logits = W.zipf_logits(w, 0, 0, T)
    x, _ = W.activations(w, 0, T)
    routed = _route(eo, logits, k)
    cnt = routed[2].cpu().numpy()
    assert cnt.max() > 128 and cnt.sum() == T * k          # multi-tile and ragged experts
    y = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_TC, H, I, E)
    ridx, rw = route.route(logits, k)
    np.testing.assert_array_equal(routed[0].cpu().numpy(), ridx)
    ref = oracle_rows(w, 0, x, ridx, rw, np.arange(T), tc=True, workers=0)
    err = report(y, ref)
    assert err <= TOL, err


def test_tc_and_gemv_paths_agree(eo, small_layer):
    w, store = small_layer
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 40
    logits = W.zipf_logits(w, 0, 5000, T)
    x, _ = W.activations(w, 5000, T)
    routed = _route(eo, logits, k)
    y_tc = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_TC, H, I, E)
    y_gv = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_GEMV, H, I, E)
    ridx, rw = route.route(logits, k)
    xv = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref_exact = moe.moe_layer(moe.ExpertCache(OraclePackedLayer(w, 0), H, I), H, I, xv, ridx, rw)
    assert report(y_gv, ref_exact) <= TOL
    # the bf16 model and the exact layer differ by the bf16 rounding of weights and h
    assert report(y_tc, ref_exact) <= 2e-2


def test_tc_path_with_host_mapped_experts(eo):
    """Every other expert in pinned host memory: the tensor-core kernels read
    those experts' bytes with plain loads over PCIe instead of TMA tiles and
    must give the same layer."""
    from expert_offload_b200.model import ExpertStore
    w = dataclasses.replace(W.WORKLOADS[4], experts=16)
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 96
    loc = (np.arange(E) % 2).astype(np.uint8)[None, :]
    slot = np.zeros((1, E), np.int64)
    for where in (0, 1):
        ids = np.nonzero(loc[0] == where)[0]
        slot[0, ids] = np.arange(len(ids))
    store = ExpertStore(torch, 1, E, H, I, device_fill(torch, w), loc=loc, slot=slot)
    try:
        logits = W.zipf_logits(w, 0, 700, T)
        x, _ = W.activations(w, 700, T)
        routed = _route(eo, logits, k)
        y = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_TC, H, I, E)
        ridx, rw = route.route(logits, k)
        assert set(ridx.ravel() % 2) == {0, 1}          # experts from both memories
        ref = oracle_rows(w, 0, x, ridx, rw, np.arange(T), tc=True, workers=0)
        err = report(y, ref)
        assert err <= TOL, err
    finally:
        store.close()


@pytest.mark.slow
def test_tc_prefill_chunk_8192_head_expert_and_sample(eo):
    """The 512-expert, 8192-token prefill chunk at full size, in the launch the
    bench times.  Compared element by element with the oracle's bf16 model:
    every token routed to the most popular expert (all of its 128-pair tiles,
    the ragged last one included) and a seeded sample of 256 other tokens.
    The oracle runs expert by expert in spawned worker processes."""
    from expert_offload_b200.model import ExpertStore
    from tests.gpu_util import oracle_rows
    w = W.WORKLOADS[4]
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 8192
    store = ExpertStore(torch, 1, E, H, I, device_fill(torch, w))
    logits = W.zipf_logits(w, 0, 0, T)
    x, _ = W.activations(w, 0, T)
    routed = _route(eo, logits, k)
    y = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_AUTO, H, I, E)
    assert np.all(np.isfinite(y))
    ridx, rw = route.route(logits, k)
    np.testing.assert_array_equal(routed[0].cpu().numpy(), ridx)
    cnt = np.bincount(ridx.ravel(), minlength=E)
    head = int(np.argmax(cnt))
    head_tokens = np.nonzero((ridx == head).any(axis=1))[0]
    assert len(head_tokens) == cnt[head] and cnt[head] > 40 * 128   # dozens of tiles
    rest = np.setdiff1d(np.arange(T), head_tokens)
    sample = np.sort(np.random.default_rng(0x5EED).choice(rest, 256, replace=False))
    tokens = np.concatenate([head_tokens, sample])
    ref = oracle_rows(w, 0, x, ridx, rw, tokens, tc=True)
    err = report(y[tokens], ref)
    assert err <= TOL, err
