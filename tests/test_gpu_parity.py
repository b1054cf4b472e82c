"""GPU parity: the CUDA path against the oracle on the same seeded inputs.

Bit-exact for packed bytes, dequantised weights, top-k indices and grouping;
y within max relative error 1e-3 per token (fp32 accumulation); routing
weights within f32 rounding.  Outputs carry guard regions that must stay
untouched (the padding-write check of the Strata report's tuning tool,
pitfall 4)."""
import numpy as np
import pytest

import synth
from oracle import hfq4, moe, route
from synth import workloads as W
from tests.gpu_util import TOL, OraclePackedLayer, device_fill, max_rel_err

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
GUARD = 4096


@pytest.fixture(scope="module")
def eo():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    synth.build()
    from expert_offload_b200 import build
    build.build()
    import expert_offload_b200
    return expert_offload_b200


def guarded(n, dtype, fill_byte=0xA5):
    """A device buffer of n elements with guard regions on both sides."""
    esz = torch.tensor([], dtype=dtype).element_size()
    g = GUARD // esz
    raw = torch.full(((n + 2 * g) * esz,), fill_byte, dtype=torch.uint8, device="cuda")
    return raw, raw.view(dtype)[g:g + n]


def assert_guards(raw, n_bytes):
    r = raw.cpu().numpy()
    assert np.all(r[:GUARD] == 0xA5) and np.all(r[GUARD + n_bytes:] == 0xA5), "write outside output"


def ws(n):
    return torch.zeros(max(n, 256), dtype=torch.uint8, device="cuda")


# ------------------------------------------------------------ generators

def test_synth_bits_agree_host_and_device(eo):
    out = torch.empty((3, 128, 256), dtype=torch.float32, device="cuda")
    synth.weights_dev(out.data_ptr(), 0x1234, 5, 7, 3, synth.MAT_UP, 128, 256, 0.02,
                      torch.cuda.current_stream().cuda_stream)
    ref = synth.weights(0x1234, 5, 7, 3, synth.MAT_UP, 128, 256, 0.02)
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ---------------------------------------------------------------- packing

@pytest.mark.parametrize("E,H,I", [(16, 256, 128), (2, 2048, 512), (3, 384, 640)])
def test_device_pack_is_bit_identical_to_oracle(eo, E, H, I):
    rng = np.random.default_rng(H + I)
    g = (rng.standard_normal((E, I, H)) * 0.02).astype(np.float32)
    u = (rng.standard_normal((E, I, H)) * 0.02).astype(np.float32)
    d = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    g[0, 0] = 0.25                                   # constant row
    eb = hfq4.expert_bytes(H, I)
    raw, out = guarded(E * eb, torch.uint8)
    eo.hfq4_pack_experts_device(torch.from_numpy(g).cuda(), torch.from_numpy(u).cuda(),
                                torch.from_numpy(d).cuda(), out, E, H, I)
    torch.cuda.synchronize()
    ref = np.concatenate([hfq4.pack_expert(g[e], u[e], d[e]) for e in range(E)])
    np.testing.assert_array_equal(out.cpu().numpy(), ref)
    assert_guards(raw, E * eb)


@pytest.mark.parametrize("rows,cols", [(7, 256), (5, 384), (3, 2048), (256, 128), (1, 8192)])
def test_dequant_is_bit_identical_to_oracle(eo, rows, cols):
    w = (np.random.default_rng(rows * cols).standard_normal((rows, cols)) * 0.02).astype(np.float32)
    packed = hfq4.quantize_matrix(w)
    raw, out = guarded(rows * cols, torch.float32)
    eo.hfq4_dequant(torch.from_numpy(packed).cuda(), rows, cols, out)
    torch.cuda.synchronize()
    ref = hfq4.dequantize_f32(packed, rows, cols)
    np.testing.assert_array_equal(out.cpu().numpy().reshape(rows, cols).view(np.uint32),
                                  ref.view(np.uint32))
    assert_guards(raw, rows * cols * 4)


# ------------------------------------------------------------------ route

def _route_gpu(eo, logits, k, group):
    T, E = logits.shape
    lg = torch.from_numpy(np.ascontiguousarray(logits)).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    if group:
        cnt = torch.empty(E, dtype=torch.int32, device="cuda")
        off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
        w = ws(eo.hfq_route_workspace_bytes(T, E, k))
        eo.moe_route(lg, T, E, k, idx, wts, cnt, off, perm, w)
        torch.cuda.synchronize()
        return (idx.cpu().numpy(), wts.cpu().numpy(), cnt.cpu().numpy(), off.cpu().numpy(),
                perm.cpu().numpy())
    eo.moe_route(lg, T, E, k, idx, wts)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), wts.cpu().numpy()


def _check_route(eo, logits, k, group=True):
    got = _route_gpu(eo, logits, k, group)
    ridx, rw = route.route(logits, k)
    np.testing.assert_array_equal(got[0], ridx)
    np.testing.assert_allclose(got[1], rw, rtol=2e-6, atol=1e-7)
    if group:
        cnt, off, perm = route.group_by_expert(ridx, logits.shape[1])
        np.testing.assert_array_equal(got[2], cnt)
        np.testing.assert_array_equal(got[3], off)
        np.testing.assert_array_equal(got[4], perm)


def test_route_tiny_workload(eo):
    w = W.WORKLOADS[1]
    _check_route(eo, W.logits(w, 0, 0, 8), w.top_k)


@pytest.mark.parametrize("T", [1, 2, 5, 8, 257])
def test_route_decode_and_verify_shapes(eo, T):
    w = W.WORKLOADS[3]
    _check_route(eo, W.logits(w, 7, 100, T), w.top_k)


def test_route_prefill_zipf_8192(eo):
    w = W.WORKLOADS[4]
    _check_route(eo, W.logits(w, 0, 0, 8192), w.top_k)


def test_route_ties_and_degenerate_cases(eo):
    l = np.array([[1.0, 2.0, 2.0, 0.0, 2.0, -1.0, 2.0, 0.5]], dtype=np.float32)
    _check_route(eo, l, 3)                       # three of four tied values selected
    _check_route(eo, np.full((3, 16), 0.25, np.float32), 4)   # all equal
    _check_route(eo, np.random.default_rng(1).standard_normal((4, 8)).astype(np.float32), 8)  # k = E
    _check_route(eo, np.random.default_rng(2).standard_normal((9, 512)).astype(np.float32), 16)
    _check_route(eo, np.random.default_rng(3).standard_normal((2, 1)).astype(np.float32), 1)


# ---------------------------------------------------------------- forward

def test_forward_tiny_workload_all_tokens(eo):
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[1]
    H, I, E, k, T = w.hidden, w.inter, w.experts, w.top_k, 8
    store = ExpertStore(torch, 1, E, H, I, device_fill(torch, w))
    oracle_layer = OraclePackedLayer(w, 0)
    for e in range(E):       # device packer at this shape, bit for bit
        np.testing.assert_array_equal(store.expert_bytes_at(0, e), oracle_layer[e])
    logits = W.logits(w, 0, 0, T)
    x, dt = W.activations(w, 0, T)
    idx, wts = _route_gpu(eo, logits, k, False)
    ridx, rw = route.route(logits, k)
    np.testing.assert_array_equal(idx, ridx)
    raw, y = guarded(T * H, torch.float32)
    rawb, yb = guarded(T * H, torch.bfloat16)
    wsb = ws(eo.hfq4_moe_workspace_bytes(T, k, H, I, E))
    eo.hfq4_moe_forward(store.layers[0], torch.from_numpy(x).cuda(), eo.HFQ_F32, T,
                        torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), k, y, wsb,
                        y_bf16=yb)
    torch.cuda.synchronize()
    ref = moe.moe_layer(oracle_layer, H, I, x.astype(np.float64), ridx, rw)
    err = max_rel_err(y.cpu().numpy(), ref)
    assert err <= TOL, err
    # bf16 output: within one bf16 step of the oracle's value
    yb32 = yb.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(yb32 - ref) <= np.abs(ref) * 2**-7 + 1e-30)
    assert_guards(raw, T * H * 4)
    assert_guards(rawb, T * H * 2)


@pytest.fixture(scope="module")
def decode_layer(eo):
    """Layer 3 of the 256-expert decode workload, resident on the device."""
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[2]
    fill = device_fill(torch, w)
    store = ExpertStore(torch, 1, w.experts, w.hidden, w.inter,
                        lambda l, g, u, d: fill(3, g, u, d))
    return w, store


@pytest.mark.parametrize("T", [1, 3, 8])
def test_forward_decode_shape(eo, decode_layer, T):
    w, store = decode_layer
    H, I, E, k = w.hidden, w.inter, w.experts, w.top_k
    logits = W.logits(w, 3, 500, T)
    x, _ = W.activations(w, 500, T)
    ridx, rw = route.route(logits, k)
    idx, wts = _route_gpu(eo, logits, k, False)
    np.testing.assert_array_equal(idx, ridx)
    oracle_layer = OraclePackedLayer(w, 3)
    for e in sorted(set(ridx.ravel().tolist()))[:4]:
        np.testing.assert_array_equal(store.expert_bytes_at(0, e), oracle_layer[e])
    raw, y = guarded(T * H, torch.float32)
    wsb = ws(eo.hfq4_moe_workspace_bytes(T, k, H, I, E))
    eo.hfq4_moe_forward(store.layers[0], torch.from_numpy(x.view(np.int16)).cuda(), eo.HFQ_BF16,
                        T, torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), k, y, wsb)
    torch.cuda.synchronize()
    ref = moe.moe_layer(oracle_layer, H, I, synth.bf16_bits_to_f32(x).astype(np.float64), ridx, rw)
    err = max_rel_err(y.cpu().numpy(), ref)
    assert err <= TOL, err
    assert_guards(raw, T * H * 4)


# ------------------------------------------------------------ decode stack

@pytest.mark.slow
def test_decode_stack_full_workload(eo):
    """The 40-layer, 256-expert decode stack at T = 1, in the launch the bench
    times, against the oracle's own residual chain."""
    from expert_offload_b200.model import ExpertStore
    w = W.WORKLOADS[2]
    H, I, E, k, L, T = w.hidden, w.inter, w.experts, w.top_k, w.layers, 1
    store = ExpertStore(torch, L, E, H, I, device_fill(torch, w))
    logits = W.logits_stack(w, 0, T)                             # [L, T, E]
    x0, _ = W.activations(w, 0, T)
    d_logits = torch.from_numpy(logits).cuda()
    d_x0 = torch.from_numpy(x0.view(np.int16)).cuda()
    x_out = torch.empty((T, H), dtype=torch.int16, device="cuda")
    y_all = torch.empty((L, T, H), dtype=torch.float32, device="cuda")
    idx_all = torch.empty((L, T, k), dtype=torch.int32, device="cuda")
    wts_all = torch.empty((L, T, k), dtype=torch.float32, device="cuda")
    wsb = ws(eo.hfq4_stack_workspace_bytes(T, k, H, I, E))
    eo.hfq4_moe_decode_stack(store.layers, d_logits, k, d_x0, T, x_out, wsb, y_all=y_all,
                             idx_all=idx_all, wts_all=wts_all)
    torch.cuda.synchronize()
    eo.hfq_workspace_status(wsb)
    caches = [moe.ExpertCache(OraclePackedLayer(w, l), H, I) for l in range(L)]
    ys, xs = moe.residual_stack(caches, logits, synth.bf16_bits_to_f32(x0).astype(np.float64), k,
                                route.route)
    np.testing.assert_array_equal(idx_all.cpu().numpy(),
                                  np.stack([route.route(logits[l], k)[0] for l in range(L)]))
    y_gpu = y_all.cpu().numpy()
    errs = [max_rel_err(y_gpu[l], ys[l]) for l in range(L)]
    assert max(errs) <= TOL, errs
    # the bf16 residual stream: equal to the oracle's except where the oracle's
    # sum lies within the tolerance of a bf16 rounding boundary
    xg = synth.bf16_bits_to_f32(x_out.cpu().numpy().view(np.uint16)).astype(np.float64)
    diff = np.abs(xg - xs[-1])
    assert np.mean(diff > 0) < 0.01 and np.all(diff <= np.abs(xs[-1]) * 2**-6 + 1e-6)
    # spot-check the device-packed bytes of some used experts
    used = idx_all.cpu().numpy()
    for l in (0, L // 2, L - 1):
        e = int(used[l, 0, 0])
        np.testing.assert_array_equal(store.expert_bytes_at(l, e), caches[l].experts[e])
