"""The C ABI without a GPU: the library loads, exports every function that
include/*.h declares, and its host-only parts (sizes, host packer, placement,
argument checks) agree with the oracle.  No call here launches a kernel."""
import glob
import os
import re

import numpy as np
import pytest

import expert_offload_b200 as eo
from oracle import hfq4, placement

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            line = m.group(0)
            if line.startswith(("typedef", "#")):
                continue
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module", autouse=True)
def built():
    from expert_offload_b200 import build
    build.build()


def test_every_declared_symbol_is_exported_and_bound():
    declared = _declared_functions()
    assert len(declared) >= 18
    lib = eo.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(eo.symbols())


def test_sizes_match_oracle():
    for r, c in [(512, 2048), (2048, 512), (128, 256), (256, 128), (3, 300)]:
        assert eo.hfq4_matrix_bytes(r, c) == hfq4.matrix_bytes(r, c)
    for H, I in [(2048, 512), (256, 128), (384, 640)]:
        assert eo.hfq4_expert_bytes(H, I) == hfq4.expert_bytes(H, I)
    assert eo.hfq4_matrix_bytes(0, 5) == 0
    assert eo.lib().hfq_version() >= 10000


@pytest.mark.parametrize("k,H,I,E", [(8, 2048, 512, 256), (8, 2048, 512, 512), (4, 256, 128, 16),
                                     (16, 1024, 1024, 64)])
def test_one_token_workspace_holds_the_tagged_exchange_buffers(k, H, I, E):
    """The one-token kernel exchanges h and the next layer's input as 8-byte
    {value, tag} words in two buffers (layer parity): the workspace sizes the
    library reports must hold 2 x k x Ip and 2 x H such words besides the
    control block (Ip = inter padded to whole 256-weight blocks)."""
    Ip = -(-I // 256) * 256
    h_words, x_words = 2 * k * Ip, 2 * H
    assert eo.hfq4_moe_workspace_bytes(1, k, H, I, E) >= 8 * h_words
    assert eo.hfq4_stack_workspace_bytes(1, k, H, I, E) >= 8 * (h_words + x_words)
    # more tokens never need less
    for T in range(2, 9):
        assert eo.hfq4_stack_workspace_bytes(T, k, H, I, E) >= eo.hfq4_stack_workspace_bytes(T - 1, k, H, I, E)
        assert eo.hfq4_stack_workspace_bytes(T, k, H, I, E) % 256 == 0


@pytest.mark.parametrize("E,H,I", [(2, 256, 128), (1, 512, 256), (3, 384, 640)])
def test_host_pack_is_bit_identical_to_oracle(E, H, I):
    rng = np.random.default_rng(E * H + I)
    g = (rng.standard_normal((E, I, H)) * 0.02).astype(np.float32)
    u = (rng.standard_normal((E, I, H)) * 0.02).astype(np.float32)
    d = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    g[0, 0, :] = 0.5                       # a constant row (scale 0)
    g[0, 1, :256] = np.float32(-0.25) + np.float32(0.0625) * (np.arange(256) % 16)   # exact grid
    eb = hfq4.expert_bytes(H, I)
    out = np.zeros(E * eb, dtype=np.uint8)
    eo.hfq4_pack_experts(g, u, d, out, E, H, I)
    ref = np.concatenate([hfq4.pack_expert(g[e], u[e], d[e]) for e in range(E)])
    np.testing.assert_array_equal(out, ref)


def test_host_pack_rejects_small_output():
    g = np.zeros((1, 128, 256), np.float32)
    out = np.zeros(10, np.uint8)
    with pytest.raises(eo.HfqError) as e:
        eo.hfq4_pack_experts(g, g, g.transpose(0, 2, 1).copy(), out, 1, 256, 128)
    assert e.value.status == -1 and "needed" in e.value.message


@pytest.mark.parametrize("N,h", [(0, 0), (2, 0), (1, 2), (-1, 3), (-1, 0), (4, 1)])
def test_placement_matches_oracle(N, h):
    rng = np.random.default_rng(N * 10 + h + 100)
    counts = rng.integers(0, 20, (4, 9)).astype(np.uint32)
    counts[1, 3] = counts[1, 5] = counts[1].max() + 1      # a tie in the hot ranking
    eb = 1000
    budget = 17_500
    ref = placement.place(counts, eb, N, h, budget)
    if ref.ok:
        loc, slot, hn, hs = eo.hfq_placement_build(counts, eb, N, h, budget)
        np.testing.assert_array_equal(loc, ref.loc)
        np.testing.assert_array_equal(slot, ref.slot)
        assert (hn, hs) == (ref.hbm_needed, ref.host_needed)
    else:
        with pytest.raises(eo.HfqError) as e:
            eo.hfq_placement_build(counts, eb, N, h, budget)
        assert e.value.status == -4
        assert "DOES NOT FIT" in e.value.message and f"deficit {ref.deficit}" in e.value.message
        assert e.value.hbm_needed == ref.hbm_needed


def test_placement_pointers():
    loc = np.array([[0, 1], [1, 0]], np.uint8)
    slot = np.array([[0, 0], [1, 1]], np.int64)
    p = eo.hfq_placement_pointers(loc, slot, 100, 0x10000, 0x90000)
    assert p.tolist() == [[0x10000, 0x90000], [0x90000 + 100, 0x10000 + 100]]


def test_argument_errors_are_caught_before_launch():
    lib = eo.lib()
    assert lib.moe_route(None, 1, 16, 4, None, None, None, None, None, None, 0, None) == -1
    assert lib.moe_route(1024, 1, 600, 4, 1024, 1024, None, None, None, None, 0, None) == -3
    assert lib.moe_route(1024, 1, 16, 17, 1024, 1024, None, None, None, None, 0, None) == -3
    assert lib.moe_route(1024, 4, 16, 4, 1024, 1024, 1024, None, None, None, 0, None) == -1
    assert lib.moe_route(1024, 4096, 16, 4, 1024, 1024, 1024, 1024, 1024, None, 0, None) == -8
    lay = eo.Layer(1024, 16, 256, 100)                          # inter not a multiple of 128
    assert lib.hfq4_moe_forward(eo.ctypes.byref(lay.struct), 1024, 0, 1, 1024, 1024, 4, None,
                                None, None, 1024, None, 0, 1024, 1 << 20, None) == -3
    lay = eo.Layer(1024, 16, 256, 128)
    assert lib.hfq4_moe_forward(eo.ctypes.byref(lay.struct), 1024, 0, 1, 1024, 1024, 4, None,
                                None, None, 1024, None, 0, 1024, 16, None) == -8   # workspace
    assert lib.hfq4_moe_forward(eo.ctypes.byref(lay.struct), 1028, 0, 1, 1024, 1024, 4, None,
                                None, None, 1024, None, 0, 1024, 1 << 20, None) == -2  # align
    assert "16-byte" in eo.last_error()
    assert lib.hfq4_dequant(1028, 1, 256, 1024, None) == -2
    assert lib.hfq_host_arena_destroy(12345) == -1


def test_placement_hand_worked_cases():
    """The library's placement on the hand-worked cases of
    tests/golden/placement_auto.txt (40 layers x 256 experts of 1,671,168 bytes)."""
    from tests.golden_io import load_placement_cases
    L, E, eb = 40, 256, 1_671_168
    counts = np.tile(np.arange(E, dtype=np.uint32), (L, 1))
    for c in load_placement_cases():
        if c["ok"]:
            loc, slot, hn, hs = eo.hfq_placement_build(counts, eb, c["resident"], c["hot"], c["budget"])
            assert (hn, hs) == (c["hbm"], c["host"]), c["name"]
            assert int((loc[:, :] == 0).all(axis=1).sum()) == c["N"], c["name"]
        else:
            with pytest.raises(eo.HfqError) as e:
                eo.hfq_placement_build(counts, eb, c["resident"], c["hot"], c["budget"])
            assert e.value.status == -4, c["name"]
            assert f"deficit {c['deficit']}" in e.value.message, c["name"]
            assert (e.value.hbm_needed, e.value.host_needed) == (c["hbm"], c["host"]), c["name"]


def test_host_arena_refuses_an_impossible_size():
    """Allocation failure of the pinned expert arena is reported as
    HFQ_ERR_ALLOC with the byte count, for both page-size choices (no GPU
    needed: the request fails before any device is involved or at the
    registration)."""
    huge = 1 << 60
    for flags in (0, eo.ARENA_HUGEPAGE):
        with pytest.raises(eo.HfqError) as e:
            eo.hfq_host_arena_create(huge, flags)
        assert e.value.status == -7
        assert str(huge) in e.value.message


def test_router_argument_errors_are_caught_before_launch():
    """moe_router_logits and the routed decode stack refuse bad arguments on
    the host (no kernel is launched on these paths)."""
    lib = eo.lib()
    bf16, f32 = eo.HFQ_BF16, eo.HFQ_F32
    assert lib.moe_router_logits(None, bf16, 1, 256, 1024, bf16, 16, 1024, None) == -1
    assert lib.moe_router_logits(1024, 7, 1, 256, 1024, bf16, 16, 1024, None) == -1          # dtype
    assert lib.moe_router_logits(1024, bf16, 1, 252, 1024, bf16, 16, 1024, None) == -3       # hidden % 8
    assert lib.moe_router_logits(1024, bf16, 1, 256, 1024, bf16, 513, 1024, None) == -3      # experts
    assert lib.moe_router_logits(1026, bf16, 1, 256, 1024, bf16, 16, 1024, None) == -2       # alignment
    lay = eo.Layer(1024, 256, 2048, 512)
    arr = eo.layer_array([lay])
    f = lib.hfq4_moe_decode_stack_routed
    need = eo.hfq4_stack_workspace_bytes(1, 8, 2048, 512, 256)
    assert f(arr, 0, 1024, bf16, 8, 1024, 1, 2048, None, None, None, None, 1024, need, None) == -1
    assert f(arr, 1, None, bf16, 8, 1024, 1, 2048, None, None, None, None, 1024, need, None) == -1
    assert f(arr, 1, 1024, 9, 8, 1024, 1, 2048, None, None, None, None, 1024, need, None) == -1
    assert f(arr, 1, 1024, f32, 8, 1024, 9, 2048, None, None, None, None, 1024, need, None) == -3   # T
    assert f(arr, 1, 1024, bf16, 8, 1026, 1, 2048, None, None, None, None, 1024, need, None) == -2  # x0
    assert f(arr, 1, 1024, bf16, 8, 1024, 1, 2048, None, 4096, None, None, 1024, need, None) == -1  # idx without wts
    assert f(arr, 1, 1024, bf16, 8, 1024, 1, 2048, None, None, None, None, 1024, 64, None) == -8    # workspace
    # the routed stack needs room for the logit exchange and its own residual pair
    assert need > eo.hfq4_moe_workspace_bytes(1, 8, 2048, 512, 256)
