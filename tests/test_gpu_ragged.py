"""GPU parity at ragged shapes: hidden and expert intermediate sizes that are
not multiples of the 256-weight HFQ4 block (rows padded to whole blocks, pad
elements stored as q = 0 and counting as zero), through every path the
forward takes for them: the persistent kernels (1..8 tokens), the per-layer
GEMV kernels (40 tokens) and the tensor-core path (40 and 300 tokens, with
rows of an even number of blocks)."""
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
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    synth.build()
    from expert_offload_b200 import build
    build.build()
    import expert_offload_b200
    return expert_offload_b200


@pytest.fixture(scope="module")
def ragged(eo):
    """16 experts, hidden 384 (1.5 blocks per gate/up row), intermediate 640
    (2.5 blocks per down row), top-4, Zipf routing, bf16 activations."""
    from expert_offload_b200.model import ExpertStore
    w = dataclasses.replace(W.WORKLOADS[4], hidden=384, inter=640, experts=16, top_k=4)
    store = ExpertStore(torch, 1, w.experts, w.hidden, w.inter, device_fill(torch, w))
    return w, store


def _route(eo, logits, k):
    T, E = logits.shape
    lg = torch.from_numpy(np.ascontiguousarray(logits)).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    rws = torch.zeros(max(256, eo.hfq_route_workspace_bytes(T, E, k)), dtype=torch.uint8, device="cuda")
    eo.moe_route(lg, T, E, k, idx, wts, cnt, off, perm, rws)
    return idx, wts, cnt, off, perm


def _forward(eo, layer, x_bits, T, k, routed, path, H, I, E, grouped):
    idx, wts, cnt, off, perm = routed
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    need = eo.hfq4_moe_workspace_bytes(T, k, H, I, E) * (2 if path == eo.PATH_TC and T <= 8 else 1)
    ws = torch.zeros(max(256, need), dtype=torch.uint8, device="cuda")
    kw = dict(cnt=cnt, off=off, perm=perm) if grouped else {}
    eo.hfq4_moe_forward(layer, torch.from_numpy(x_bits.view(np.int16)).cuda(), eo.HFQ_BF16, T, idx,
                        wts, k, y, ws, path=path, **kw)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(ws)
    return y.cpu().numpy()


def test_ragged_experts_pack_like_the_oracle(eo, ragged):
    w, store = ragged
    oracle_layer = OraclePackedLayer(w, 0)
    for e in (0, 7, 15):
        np.testing.assert_array_equal(store.expert_bytes_at(0, e), oracle_layer[e])


@pytest.mark.parametrize("T", [1, 3, 8])
def test_ragged_persistent_kernels(eo, ragged, T):
    w, store = ragged
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    logits = W.zipf_logits(w, 0, 100, T)
    x, _ = W.activations(w, 100, T)
    routed = _route(eo, logits, k)
    ridx, rw = route.route(logits, k)
    np.testing.assert_array_equal(routed[0].cpu().numpy(), ridx)
    y = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_AUTO, H, I, E, grouped=False)
    ref = moe.moe_layer(OraclePackedLayer(w, 0), H, I, synth.bf16_bits_to_f32(x).astype(np.float64), ridx, rw)
    err = report(y, ref)
    assert err <= TOL, err


def test_ragged_gemv_path(eo, ragged):
    w, store = ragged
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 40
    logits = W.zipf_logits(w, 0, 300, T)
    x, _ = W.activations(w, 300, T)
    routed = _route(eo, logits, k)
    ridx, rw = route.route(logits, k)
    xv = synth.bf16_bits_to_f32(x).astype(np.float64)
    y_gv = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_GEMV, H, I, E, grouped=False)
    ref_exact = moe.moe_layer(moe.ExpertCache(OraclePackedLayer(w, 0), H, I), H, I, xv, ridx, rw)
    assert report(y_gv, ref_exact) <= TOL


def test_ragged_shape_without_whole_16_byte_rows_refuses_the_tensor_cores(eo, ragged):
    """inter 640 = 3 blocks per down row (408 bytes): no tensor map can step
    over such rows, so a forced tensor-core call is refused and AUTO takes the
    GEMV kernels."""
    w, store = ragged
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 40
    x, _ = W.activations(w, 300, T)
    routed = _route(eo, W.zipf_logits(w, 0, 300, T), k)
    with pytest.raises(Exception, match="even number"):
        _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_TC, H, I, E, grouped=True)
    y = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_AUTO, H, I, E, grouped=True)
    ridx, rw = route.route(W.zipf_logits(w, 0, 300, T), k)
    ref = moe.moe_layer(moe.ExpertCache(OraclePackedLayer(w, 0), H, I), H, I,
                        synth.bf16_bits_to_f32(x).astype(np.float64), ridx, rw)
    assert report(y, ref) <= TOL


@pytest.fixture(scope="module")
def ragged_tc(eo):
    """16 experts, hidden 384 (1.5 blocks per gate/up row, padded to 2),
    intermediate 896 (3.5 blocks per down row, padded to 4): partial K
    blocks and a partial last raw load on the tensor-core path."""
    from expert_offload_b200.model import ExpertStore
    w = dataclasses.replace(W.WORKLOADS[4], hidden=384, inter=896, experts=16, top_k=4)
    store = ExpertStore(torch, 1, w.experts, w.hidden, w.inter, device_fill(torch, w))
    return w, store


@pytest.mark.parametrize("T", [40, 300])
def test_ragged_tensor_core_path(eo, ragged_tc, T):
    w, store = ragged_tc
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    logits = W.zipf_logits(w, 0, 300, T)
    x, _ = W.activations(w, 300, T)
    routed = _route(eo, logits, k)
    ridx, rw = route.route(logits, k)
    xv = synth.bf16_bits_to_f32(x).astype(np.float64)
    y_tc = _forward(eo, store.layers[0], x, T, k, routed, eo.PATH_TC, H, I, E, grouped=True)
    ref_tc = oracle_rows(w, 0, x, ridx, rw, np.arange(T), tc=True, workers=0)
    err = report(y_tc, ref_tc)
    assert err <= TOL, err
