"""Pins for the oracle's HFQ4 format (no GPU).

The pages print no packed example, so the pins are by construction: blocks
packed by hand (tests/golden/hfq4_handpacked.txt), invariants that any
correct min/max 4-bit quantiser satisfies, and planted mistakes that at least
one pin must catch.
"""
import numpy as np
import pytest

from oracle import hfq4
from tests.golden_io import load_hfq4_cases

CASES = load_hfq4_cases()


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_handpacked_blocks_dequantise_to_hand_values(case):
    R, C = case["rows"], case["cols"]
    assert len(case["bytes"]) == hfq4.matrix_bytes(R, C)
    w = hfq4.dequantize_exact(case["bytes"], R, C)
    np.testing.assert_array_equal(w, case["expect"])


def test_sizes():
    assert hfq4.BLOCK_BYTES == 136 and hfq4.BLOCK == 256
    assert hfq4.matrix_bytes(512, 2048) == 512 * 8 * 136 == 557_056
    assert hfq4.matrix_bytes(2048, 512) == 557_056
    assert hfq4.expert_bytes(2048, 512) == 1_671_168
    assert 256 * hfq4.expert_bytes(2048, 512) == 408 * 2**20      # 408 MiB per layer
    assert hfq4.matrix_bytes(256, 128) == 256 * 136                # padded down of the tiny layer
    assert hfq4.expert_bytes(256, 128) == 69_632


def test_repack_of_handpacked_is_identity():
    for c in CASES:
        s, z, q = hfq4.unpack_blocks(c["bytes"], c["rows"], c["cols"])
        np.testing.assert_array_equal(hfq4.pack_blocks(s, z, q), c["bytes"])


def _rand(shape, seed, sigma=0.02):
    return (np.random.default_rng(seed).standard_normal(shape) * sigma).astype(np.float32)


@pytest.mark.parametrize("shape", [(3, 256), (4, 512), (5, 300), (2, 128), (1, 1)])
def test_quantiser_invariants(shape):
    w = _rand(shape, 1)
    R, C = shape
    s, z, q = hfq4.quantize_blocks(w)
    nb = hfq4.blocks_per_row(C)
    assert q.min() >= 0 and q.max() <= 15
    deq = hfq4.dequantize_exact(hfq4.pack_blocks(s, z, q), R, C)
    pad = np.zeros((R, nb * 256), dtype=np.float32)
    pad[:, :C] = w
    for r in range(R):
        for b in range(nb):
            lo, hi = b * 256, min((b + 1) * 256, C)
            blk = w[r, lo:hi].astype(np.float64)
            # zero is the block minimum, the minimum element has q = 0 and
            # dequantises to it exactly; the maximum has q = 15
            assert z[r, b] == np.float32(blk.min())
            assert q[r, lo + int(np.argmin(blk))] == 0
            assert deq[r, lo + int(np.argmin(blk))] == blk.min()
            if hi - lo > 1 and blk.max() > blk.min():
                assert q[r, lo + int(np.argmax(blk))] == 15
            # pad elements are q = 0
            assert np.all(q[r, hi:(b + 1) * 256] == 0)
            # reconstruction error is at most half a step (plus f32 rounding of the step)
            err = np.abs(deq[r, lo:hi] - blk)
            assert np.all(err <= 0.5 * float(s[r, b]) * (1 + 2**-20) + 1e-12)


def test_scale_is_f32_range_over_15():
    w = _rand((2, 256), 7)
    s, z, _ = hfq4.quantize_blocks(w)
    for r in range(2):
        d = np.float32(np.float32(w[r].max()) - np.float32(w[r].min()))
        assert s[r, 0] == np.float32(d / np.float32(15))


def test_constant_block_is_exact():
    w = np.full((2, 256), 0.0123, dtype=np.float32)
    s, z, q = hfq4.quantize_blocks(w)
    assert np.all(s == 0) and np.all(q == 0)
    np.testing.assert_array_equal(hfq4.dequantize_f32(hfq4.pack_blocks(s, z, q), 2, 256), w)


def test_pad_does_not_enter_min_max():
    w = np.linspace(1.0, 2.0, 128, dtype=np.float32)[None, :]    # all positive
    s, z, q = hfq4.quantize_blocks(w)
    assert z[0, 0] == np.float32(1.0)                            # not 0 from the pad
    assert s[0, 0] == np.float32(np.float32(1.0) / np.float32(15))


def test_requantising_dequantised_weights_is_a_fixed_point():
    w = _rand((6, 512), 3)
    s, z, q = hfq4.quantize_blocks(w)
    deq = hfq4.dequantize_f32(hfq4.pack_blocks(s, z, q), 6, 512)
    s2, z2, q2 = hfq4.quantize_blocks(deq)
    np.testing.assert_array_equal(q2, q)
    np.testing.assert_array_equal(z2, z)
    assert np.all(np.abs(s2.astype(np.float64) - s) <= np.spacing(s) * 1.0)


def test_exact_grid_values_quantise_exactly():
    # weights already on a 15-step grid with f32-exact steps round-trip bit for bit
    q0 = np.random.default_rng(5).integers(0, 16, size=(2, 256))
    q0[:, 0], q0[:, 1] = 0, 15
    w = (-0.5 + 0.0625 * q0).astype(np.float32)
    s, z, q = hfq4.quantize_blocks(w)
    assert np.all(s == np.float32(0.0625)) and np.all(z == np.float32(-0.5))
    np.testing.assert_array_equal(q, q0)


def test_half_step_rounds_to_even():
    # (w - zero)/scale exactly k + 1/2 rounds to the even neighbour
    w = np.zeros((1, 256), dtype=np.float32)
    w[0, 1] = 15.0           # max -> scale 1, zero 0
    w[0, 2] = 2.5            # -> 2
    w[0, 3] = 3.5            # -> 4
    _, _, q = hfq4.quantize_blocks(w)
    assert q[0, 2] == 2 and q[0, 3] == 4


# --- planted mistakes: each must be caught by one of the pins above --------

def _swap_nibbles(data, rows, cols):
    s, z, q = _orig_unpack(data, rows, cols)
    q2 = q.copy()
    q2[:, 0::2], q2[:, 1::2] = q[:, 1::2], q[:, 0::2]
    return s, z, q2


_orig_unpack = hfq4.unpack_blocks


def test_planted_nibble_swap_is_caught(monkeypatch):
    monkeypatch.setattr(hfq4, "unpack_blocks", _swap_nibbles)
    c = CASES[0]
    w = hfq4.dequantize_exact(c["bytes"], c["rows"], c["cols"])
    assert not np.array_equal(w, c["expect"])


def test_planted_field_swap_is_caught(monkeypatch):
    def swapped(data, rows, cols):
        s, z, q = _orig_unpack(data, rows, cols)
        return z, s, q
    monkeypatch.setattr(hfq4, "unpack_blocks", swapped)
    c = CASES[0]
    assert not np.array_equal(hfq4.dequantize_exact(c["bytes"], c["rows"], c["cols"]), c["expect"])
