"""The router on the GPU: logits = Wr x (hipfire offload explainer, opening
section: each token's router picks its layer's top-8 experts), alone and
inside the routed decode stack, where layer l's logits come from the
residual stream x_l that the previous layers wrote.

* moe_router_logits against the oracle's fp64 logits, within the a-priori
  bound of an f32 dot product of H terms, |err| <= (H + 1) u sum_c |x_c w_c|
  (u = 2^-24; bf16 x bf16 products are exact in f32, f32 router products add
  one rounding each);
* the fused router of the one-token kernel gives the same bits as
  moe_router_logits on the same x_l;
* the routed stack against the oracle's chain (router -> route -> experts ->
  bf16 residual), compared exactly for as long as the two chains agree: the
  selection must match unless the oracle's k-th and (k+1)-th exact logits lie
  within twice the logit bound (then either selection is correct and the
  chains may part), and the residual must match unless it lands on a bf16
  rounding boundary within the y error.
"""
import numpy as np
import pytest

import synth
from oracle import moe, route
from synth import workloads as W
from tests.gpu_util import TOL, OraclePackedLayer, device_fill, report

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
U = 2.0 ** -24


@pytest.fixture(scope="module")
def eo():
    assert torch.cuda.is_available()
    synth.build()
    from expert_offload_b200 import build
    build.build()
    import expert_offload_b200
    return expert_offload_b200


def _router(w, L, bf16):
    """Router weights [L, E, H]: f32 draws, or their bf16 rounding (bits)."""
    wr = np.stack([W.router_weights(w, l) for l in range(L)]).astype(np.float32)
    if bf16:
        bits = synth.to_bf16_bits(wr)
        return bits, synth.bf16_bits_to_f32(bits).astype(np.float64)
    return wr, wr.astype(np.float64)


def _logit_bound(x, wr):
    """(H + 1) u sum_c |x_c w_ec| for x [T, H], wr [E, H] -> [T, E]."""
    return (x.shape[1] + 1) * U * (np.abs(x) @ np.abs(wr).T)


@pytest.mark.parametrize("x_bf16", [True, False], ids=["x_bf16", "x_f32"])
@pytest.mark.parametrize("r_bf16", [True, False], ids=["router_bf16", "router_f32"])
def test_router_logits_against_the_oracle(eo, x_bf16, r_bf16):
    w = W.WORKLOADS[3]                      # E 512, H 2048
    T, E, H = 5, w.experts, w.hidden
    wr_dev, wr_val = _router(w, 1, r_bf16)
    xf = W.activations_f32(w, 40, T)
    if x_bf16:
        xb = synth.to_bf16_bits(xf)
        x_dev, x_val = xb.view(np.int16), synth.bf16_bits_to_f32(xb).astype(np.float64)
    else:
        x_dev, x_val = xf, xf.astype(np.float64)
    d_x = torch.from_numpy(np.ascontiguousarray(x_dev)).cuda()
    d_wr = torch.from_numpy(np.ascontiguousarray(wr_dev[0].view(np.int16) if r_bf16 else wr_dev[0])).cuda()
    out = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    eo.moe_router_logits(d_x, eo.HFQ_BF16 if x_bf16 else eo.HFQ_F32, T, H, d_wr,
                         eo.HFQ_BF16 if r_bf16 else eo.HFQ_F32, E, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    ref = route.router_logits(x_val, wr_val[0])
    bound = _logit_bound(x_val, wr_val[0])
    err = np.abs(got - ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    print(f"router logits: max |err| / bound = {np.max(err / bound):.3e}")
    # deterministic: a second call gives the same bits
    out2 = torch.empty_like(out)
    eo.moe_router_logits(d_x, eo.HFQ_BF16 if x_bf16 else eo.HFQ_F32, T, H, d_wr,
                         eo.HFQ_BF16 if r_bf16 else eo.HFQ_F32, E, out2)
    assert torch.equal(out.view(torch.int32), out2.view(torch.int32))


def test_router_logits_rejects_bad_arguments(eo):
    x = torch.zeros((1, 256), dtype=torch.int16, device="cuda")
    wr = torch.zeros((16, 256), dtype=torch.int16, device="cuda")
    out = torch.zeros((1, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(eo.HfqError):
        eo.moe_router_logits(x, eo.HFQ_BF16, 1, 252, wr, eo.HFQ_BF16, 16, out)     # hidden % 8
    with pytest.raises(eo.HfqError):
        eo.moe_router_logits(x, eo.HFQ_BF16, 1, 256, wr, eo.HFQ_BF16, 513, out)    # too many experts
    with pytest.raises(eo.HfqError) as e:
        eo.moe_router_logits(x.data_ptr() + 2, eo.HFQ_BF16, 1, 256, wr, eo.HFQ_BF16, 16, out)
    assert e.value.status == -2            # HFQ_ERR_ALIGN


@pytest.fixture(scope="module", params=[2, 3, 1], ids=["decode_e256", "verify_e512", "tiny_e16"])
def stack_model(eo, request):
    """A prefix of a model, resident in HBM: the 40-layer decode model (H 2048,
    I 512, E 256, top-8; 4 layers), the 48-layer verify model (E 512: up to 4
    router rows per CTA; 3 layers) and the tiny layer (H 256, I 128, E 16,
    top-4: most CTAs own no router row)."""
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[request.param]
    L = min({2: 4, 3: 3, 1: 1}[request.param], w.layers)
    store = ExpertStore(torch, L, w.experts, w.hidden, w.inter, device_fill(torch, w))
    caches = [moe.ExpertCache(OraclePackedLayer(w, l), w.hidden, w.inter) for l in range(L)]
    yield w, L, store, caches
    store.close()


def _residual_chain(x0_val, y_gpu):
    """The launch's own residual stream rebuilt from its y (same f32 add and
    bf16 rounding as the kernel): [L + 1, T, H] bf16 values."""
    xs = [x0_val.astype(np.float32)]
    for y in y_gpu:
        xs.append(moe.round_bf16((xs[-1] + y.astype(np.float32)).astype(np.float64)).astype(np.float32))
    return np.stack(xs)


def _oracle_chain(L, k, x0_val, wr_val, caches):
    """The oracle's own chain: per layer (x_l, exact logits, idx, wts, y_l),
    x_{l+1} = bf16(x_l + y_l)."""
    H = x0_val.shape[1]
    x_o, out = x0_val.astype(np.float64), []
    for l in range(L):
        lo = route.router_logits(x_o, wr_val[l])
        idx_o, wts_o = route.route(lo, k)
        y_o = moe.moe_layer(caches[l], H, caches[l].inter, x_o, idx_o, wts_o)
        out.append((x_o, lo, idx_o, y_o))
        x_o = moe.round_bf16(x_o + y_o)
    return out, x_o


def _check_layer(name, l, k, x_o, lo, idx_o, y_o, wr_l, got_logits, got_idx, got_y):
    """One layer of the launch against the oracle on the same x_l.  Returns
    False where the selection legitimately differs (a near tie)."""
    bound = _logit_bound(x_o, wr_l)
    assert np.all(np.abs(got_logits - lo) <= bound), (name, l)
    if not np.array_equal(got_idx, idx_o):
        rows = np.any(got_idx != idx_o, axis=1)
        near = route.near_ties(lo, k, 2.0 * bound.max(axis=1))
        assert np.all(near[rows]), (name, l, "selection differs away from a near tie")
        return False
    err = report(got_y, y_o, name=f"{name}, layer {l}")
    assert err <= TOL, (name, l, err)
    return True


def _compare_chain(L, k, chain, wr_val, got_logits, got_idx, y_gpu, xs_gpu, name):
    """Oracle chain against the launch's, exactly until a legitimate parting."""
    for l in range(L):
        x_o, lo, idx_o, y_o = chain[l]
        np.testing.assert_array_equal(xs_gpu[l], x_o, err_msg=f"{name}: x_{l}")
        if not _check_layer(name + " chained", l, k, x_o, lo, idx_o, y_o, wr_val[l], got_logits[l],
                            got_idx[l], y_gpu[l]):
            print(f"{name}: chains part at layer {l} (near tie in the router)")
            return l
        x_next = moe.round_bf16(x_o + y_o)
        diff = xs_gpu[l + 1] != x_next
        if diff.any():
            a, b = x_next[diff], xs_gpu[l + 1][diff].astype(np.float64)
            assert np.all(np.abs(a - b) <= np.abs(a) * 2.0 ** -7 + 2.0 ** -133), (name, l)
            exact = (x_o + y_o)[diff]
            slack = np.abs(y_gpu[l].astype(np.float64) - y_o)[diff] + U * np.abs(exact)
            assert np.all(np.abs(exact - 0.5 * (a + b)) <= slack), (name, l)
            print(f"{name}: chains part after layer {l} (bf16 rounding boundary)")
            return l
    print(f"{name}: identical chains through layer {L - 1}")
    return L


@pytest.mark.parametrize("T,r_bf16", [(1, True), (1, False), (2, True), (5, True)],
                         ids=["t1_fused", "t1_router_f32", "t2", "t5"])
def test_routed_stack(eo, stack_model, T, r_bf16):
    w, L, store, caches = stack_model
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    wr_dev, wr_val = _router(w, L, r_bf16)
    x0 = synth.to_bf16_bits(W.activations_f32(w, 300, T))       # bf16 residual stream
    x0_val = synth.bf16_bits_to_f32(x0)
    d_x0 = torch.from_numpy(x0.view(np.int16)).cuda()
    d_wr = torch.from_numpy(np.ascontiguousarray(wr_dev.view(np.int16) if r_bf16 else wr_dev)).cuda()
    x_out = torch.empty((T, H), dtype=torch.int16, device="cuda")
    y_all = torch.empty((L, T, H), dtype=torch.float32, device="cuda")
    idx_all = torch.empty((L, T, k), dtype=torch.int32, device="cuda")
    wts_all = torch.empty((L, T, k), dtype=torch.float32, device="cuda")
    lg_all = torch.empty((L, T, E), dtype=torch.float32, device="cuda")
    ws = torch.zeros(eo.hfq4_stack_workspace_bytes(T, k, H, I, E), dtype=torch.uint8, device="cuda")
    rdt = eo.HFQ_BF16 if r_bf16 else eo.HFQ_F32
    for rep in range(2):              # the second call reuses the workspace (tags of a new epoch)
        eo.hfq4_moe_decode_stack_routed(store.layers, d_wr, rdt, k, d_x0, T, x_out, ws, y_all=y_all,
                                        idx_all=idx_all, wts_all=wts_all, logits_all=lg_all)
        torch.cuda.synchronize()
        eo.hfq_workspace_status(ws)
        if rep == 0:
            first = (y_all.clone(), idx_all.clone(), lg_all.clone())
    for a, b in zip(first, (y_all, idx_all, lg_all)):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32)), "not deterministic"
    y_gpu, idx_gpu = y_all.cpu().numpy(), idx_all.cpu().numpy()
    lg_gpu = lg_all.cpu().numpy()
    xs_gpu = _residual_chain(x0_val, y_gpu)
    np.testing.assert_array_equal(x_out.cpu().numpy().view(np.uint16), synth.to_bf16_bits(xs_gpu[L]))
    # every layer's logits: the same bits as moe_router_logits on the launch's x_l,
    # and the launch routed on exactly those logits
    for l in range(L):
        d_xl = torch.from_numpy(synth.to_bf16_bits(xs_gpu[l]).view(np.int16)).cuda()
        ref = torch.empty((T, E), dtype=torch.float32, device="cuda")
        eo.moe_router_logits(d_xl, eo.HFQ_BF16, T, H, d_wr[l], rdt, E, ref)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(lg_gpu[l].view(np.uint32), ref.cpu().numpy().view(np.uint32))
        idx_r, _ = route.route(lg_gpu[l], k)
        np.testing.assert_array_equal(idx_gpu[l], idx_r)
    name = f"routed stack T={T} {'bf16' if r_bf16 else 'f32'} router"
    chain, _ = _oracle_chain(L, k, x0_val, wr_val, caches)
    _compare_chain(L, k, chain, wr_val, lg_gpu, idx_gpu, y_gpu, xs_gpu, name)
    # every layer alone (the same routed entry, one layer) on the oracle's own x_l
    for l in range(L):
        x_o, lo, idx_o, y_o = chain[l]
        d_xl = torch.from_numpy(synth.to_bf16_bits(x_o.astype(np.float32)).view(np.int16)).cuda()
        eo.hfq4_moe_decode_stack_routed([store.layers[l]], d_wr[l], rdt, k, d_xl, T, x_out, ws,
                                        y_all=y_all[l], idx_all=idx_all[l], wts_all=wts_all[l],
                                        logits_all=lg_all[l])
        torch.cuda.synchronize()
        eo.hfq_workspace_status(ws)
        if not _check_layer(name + " alone", l, k, x_o, lo, idx_o, y_o, wr_val[l],
                            lg_all[l].cpu().numpy(), idx_all[l].cpu().numpy(),
                            y_all[l].cpu().numpy()):
            print(f"{name}: layer {l} alone routes differently at a near tie")
