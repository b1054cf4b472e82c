"""GPU robustness: invalid routing from the caller, and exchange buffers reused
across shapes.

An expert id outside [0, E), or a grouping whose cnt/off do not describe the
T*k pairs, must never turn into an address: the kernels record HFQ_ERR_ARG in
the workspace status word (read by hfq_workspace_status), skip or neutralise
the pair, and the next call on the same workspace is correct.  Every case
here is an input the kernels' own range checks turn into that status; none
faults.  The one-token kernel's exchange tags keep 13 bits of a launch
counter, so a workspace that changes k must not serve words another layout
wrote 8192 launches earlier."""
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


@pytest.fixture(scope="module")
def layer2(eo):
    """Layer 2 of the 256-expert decode workload."""
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[2]
    store = ExpertStore(torch, 1, w.experts, w.hidden, w.inter,
                        lambda l, g, u, d: device_fill(torch, w)(2, g, u, d))
    return w, store


def _oracle(w, layer, x_bits, idx, wts):
    xv = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    return moe.moe_layer(OraclePackedLayer(w, layer), w.hidden, w.inter, xv, idx, wts)


@pytest.mark.parametrize("T", [1, 3, 16])
def test_invalid_expert_id_is_reported_and_the_workspace_recovers(eo, layer2, T):
    """T = 1: the one-token kernel; T = 3: the 2..8-token kernel; T = 16: the
    per-layer GEMV kernels.  One id of token 0 is E + 3."""
    w, store = layer2
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    logits = W.logits(w, 2, 640, T)
    x, _ = W.activations(w, 640, T)
    ridx, rw = route.route(logits, k)
    bad = ridx.astype(np.int32).copy()
    bad[0, 2] = E + 3
    ws = torch.zeros(eo.hfq4_moe_workspace_bytes(T, k, H, I, E), dtype=torch.uint8, device="cuda")
    d_x = torch.from_numpy(x.view(np.int16)).cuda()
    d_w = torch.from_numpy(rw.astype(np.float32)).cuda()
    y = torch.zeros((T, H), dtype=torch.float32, device="cuda")
    eo.hfq4_moe_forward(store.layers[0], d_x, eo.HFQ_BF16, T, torch.from_numpy(bad).cuda(), d_w, k, y,
                        ws, path=eo.PATH_GEMV)
    torch.cuda.synchronize()
    with pytest.raises(eo.HfqError) as e:
        eo.hfq_workspace_status(ws)
    assert e.value.status == -1
    eo.hfq_workspace_status(ws)                         # cleared by the read
    if T == 16:
        # the per-layer kernels skip only the token with the bad id
        ref = _oracle(w, 2, x[1:], ridx[1:], rw[1:])
        assert report(y.cpu().numpy()[1:], ref) <= TOL
    eo.hfq4_moe_forward(store.layers[0], d_x, eo.HFQ_BF16, T,
                        torch.from_numpy(ridx.astype(np.int32)).cuda(), d_w, k, y, ws,
                        path=eo.PATH_GEMV)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(ws)
    assert report(y.cpu().numpy(), _oracle(w, 2, x, ridx, rw)) <= TOL


def test_tensor_core_path_refuses_an_inconsistent_grouping(eo):
    """cnt no longer matches off: the plan gives the tensor-core kernels no
    work items, the status word says HFQ_ERR_ARG, and the next call with the
    true grouping is correct."""
    import dataclasses

    from expert_offload_b200.model import ExpertStore
    w = dataclasses.replace(W.WORKLOADS[4], experts=16)
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 64
    store = ExpertStore(torch, 1, E, H, I, device_fill(torch, w))
    logits = W.zipf_logits(w, 0, 300, T)
    x, _ = W.activations(w, 300, T)
    lg = torch.from_numpy(logits).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    rws = torch.zeros(max(256, eo.hfq_route_workspace_bytes(T, E, k)), dtype=torch.uint8,
                      device="cuda")
    eo.moe_route(lg, T, E, k, idx, wts, cnt, off, perm, rws)
    ws = torch.zeros(eo.hfq4_moe_workspace_bytes(T, k, H, I, E), dtype=torch.uint8, device="cuda")
    y = torch.zeros((T, H), dtype=torch.float32, device="cuda")
    d_x = torch.from_numpy(x.view(np.int16)).cuda()
    bad_cnt = cnt.clone()
    bad_cnt[0] += 1
    eo.hfq4_moe_forward(store.layers[0], d_x, eo.HFQ_BF16, T, idx, wts, k, y, ws, cnt=bad_cnt,
                        off=off, perm=perm, path=eo.PATH_TC)
    torch.cuda.synchronize()
    with pytest.raises(eo.HfqError) as e:
        eo.hfq_workspace_status(ws)
    assert e.value.status == -1
    eo.hfq4_moe_forward(store.layers[0], d_x, eo.HFQ_BF16, T, idx, wts, k, y, ws, cnt=cnt,
                        off=off, perm=perm, path=eo.PATH_TC)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(ws)
    ridx, rw = route.route(logits, k)
    ref = oracle_rows(w, 0, x, ridx, rw, np.arange(T), tc=True, workers=0)
    assert report(y.cpu().numpy(), ref) <= TOL


def test_one_token_workspace_reused_across_k_through_the_tag_wrap(eo, layer2):
    """One workspace: a k = 16 launch, 8191 k = 8 launches, then k = 16 again,
    whose 13-bit tag epoch equals the first launch's.  The k = 16 words that
    the k = 8 launches never wrote must not be taken for this launch's."""
    w, store = layer2
    H, I, E = w.hidden, w.inter, w.experts
    layer = store.layers[0]
    ws = torch.zeros(eo.hfq4_moe_workspace_bytes(1, 16, H, I, E), dtype=torch.uint8, device="cuda")

    def call(token, k, n=1):
        logits = W.logits(w, 2, token, 1)
        x, _ = W.activations(w, token, 1)
        ridx, rw = route.route(logits, k)
        d_x = torch.from_numpy(x.view(np.int16)).cuda()
        d_i = torch.from_numpy(ridx.astype(np.int32)).cuda()
        d_w = torch.from_numpy(rw.astype(np.float32)).cuda()
        y = torch.full((1, H), float("nan"), dtype=torch.float32, device="cuda")
        for _ in range(n):
            eo.hfq4_moe_forward(layer, d_x, eo.HFQ_BF16, 1, d_i, d_w, k, y, ws)
        torch.cuda.synchronize()
        eo.hfq_workspace_status(ws)
        return report(y.cpu().numpy(), _oracle(w, 2, x, ridx, rw))

    assert call(5000, 16) <= TOL
    assert call(5100, 8, n=8191) <= TOL
    assert call(5200, 16) <= TOL
