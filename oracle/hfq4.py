"""HFQ4 block format: quantise, pack, unpack, dequantise (oracle, fp64).

Source: the hipfire RDNA engine thread, section "HFQ quantisation format and
GEMV optimisation": a 256-weight block is stored in 136 bytes, an f32 scale,
an f32 zero point and 128 bytes of packed 4-bit data, with weights
reconstructed as w = zero + scale * q.

The pages leave open what this module fixes (each is a stated reading):
  * field order: scale, zero, nibbles, little-endian (the listing order);
  * nibble order: byte j holds element 2j in its low nibble, 2j+1 in its high;
  * a row whose length is not a multiple of 256 is padded to whole blocks; pad
    elements take no part in min/max, are stored as q = 0 and never count;
  * the quantiser is the plain asymmetric min/max one with 15 steps (the
    gfx1151 engine README, "features" section, says its converter needs no
    calibration data): scale = f32(f32(max - min) / 15), zero = min,
    q = clamp(rint_half_even(f32(f32(w - zero) / scale)), 0, 15), and a
    constant block (scale == 0) stores q = 0.

Every f32 operation of the quantiser is done with numpy float32 arithmetic,
which is IEEE single precision with round-to-nearest-even.  Dequantisation is
exact in fp64 (scale*q has at most 28 significant bits and the sum is checked
to be exact), so RN_f32 of it is the one correctly rounded f32 weight.
"""
from __future__ import annotations

import numpy as np

BLOCK = 256          # weights per block
BLOCK_BYTES = 136    # 4 (scale) + 4 (zero) + 128 (nibbles)
QMAX = 15


def blocks_per_row(cols: int) -> int:
    return (cols + BLOCK - 1) // BLOCK


def matrix_bytes(rows: int, cols: int) -> int:
    """Bytes of an HFQ4 matrix: rows x ceil(cols/256) blocks of 136 bytes."""
    return rows * blocks_per_row(cols) * BLOCK_BYTES


def expert_bytes(hidden: int, inter: int) -> int:
    """gate [I x H] + up [I x H] + down [H x I], each an HFQ4 matrix."""
    return 2 * matrix_bytes(inter, hidden) + matrix_bytes(hidden, inter)


def quantize_blocks(w: np.ndarray):
    """Quantise f32 rows into blocks.

    w: f32 [R, C].  Returns (scale f32 [R, nb], zero f32 [R, nb],
    q uint8 [R, nb*256]) with pad elements q = 0."""
    w = np.asarray(w, dtype=np.float32)
    R, C = w.shape
    nb = blocks_per_row(C)
    padded = np.zeros((R, nb * BLOCK), dtype=np.float32)
    padded[:, :C] = w
    real = np.zeros((R, nb * BLOCK), dtype=bool)
    real[:, :C] = True
    wb = padded.reshape(R, nb, BLOCK)
    rb = real.reshape(R, nb, BLOCK)
    mn = np.where(rb, wb, np.float32(np.inf)).min(axis=2).astype(np.float32)
    mx = np.where(rb, wb, np.float32(-np.inf)).max(axis=2).astype(np.float32)
    scale = (mx - mn) / np.float32(QMAX)          # two f32 ops, each rounded once
    zero = mn
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (wb - zero[:, :, None]) / scale[:, :, None]   # f32 subtract, f32 divide
    q = np.clip(np.rint(t), 0, QMAX)
    q = np.where(rb & (scale[:, :, None] != 0), q, 0).astype(np.uint8)
    return scale.astype(np.float32), zero.astype(np.float32), q.reshape(R, nb * BLOCK)


def pack_blocks(scale: np.ndarray, zero: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Lay blocks out as bytes: [R][nb][scale f32 | zero f32 | 128 nibble bytes]."""
    R, nb = scale.shape
    qb = q.reshape(R, nb, BLOCK // 2, 2).astype(np.uint8)
    nib = (qb[..., 0] & 0xF) | ((qb[..., 1] & 0xF) << 4)
    out = np.empty((R, nb, BLOCK_BYTES), dtype=np.uint8)
    out[:, :, 0:4] = np.ascontiguousarray(scale, dtype="<f4").view(np.uint8).reshape(R, nb, 4)
    out[:, :, 4:8] = np.ascontiguousarray(zero, dtype="<f4").view(np.uint8).reshape(R, nb, 4)
    out[:, :, 8:] = nib
    return out.reshape(-1)


def quantize_matrix(w: np.ndarray) -> np.ndarray:
    """f32 [R, C] -> HFQ4 bytes (uint8, matrix_bytes(R, C) long)."""
    return pack_blocks(*quantize_blocks(w))


def unpack_blocks(data: np.ndarray, rows: int, cols: int):
    """Inverse of pack_blocks: (scale f32 [R,nb], zero f32 [R,nb], q uint8 [R, nb*256])."""
    nb = blocks_per_row(cols)
    b = np.asarray(data, dtype=np.uint8)[: matrix_bytes(rows, cols)].reshape(rows, nb, BLOCK_BYTES)
    scale = np.ascontiguousarray(b[:, :, 0:4]).view("<f4").reshape(rows, nb).astype(np.float32)
    zero = np.ascontiguousarray(b[:, :, 4:8]).view("<f4").reshape(rows, nb).astype(np.float32)
    nib = b[:, :, 8:]
    q = np.empty((rows, nb, BLOCK), dtype=np.uint8)
    q[:, :, 0::2] = nib & 0xF
    q[:, :, 1::2] = nib >> 4
    return scale, zero, q.reshape(rows, nb * BLOCK)


def _two_sum_error(a: np.ndarray, b: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Rounding error of s = fl(a + b) (Knuth's TwoSum), exactly."""
    bb = s - a
    return (a - (s - bb)) + (b - bb)


def dequantize_exact(data: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """w = zero + scale*q for every real element, exactly, as f64 [R, C]."""
    scale, zero, q = unpack_blocks(data, rows, cols)
    nb = scale.shape[1]
    s = np.repeat(scale.astype(np.float64), BLOCK, axis=1)
    z = np.repeat(zero.astype(np.float64), BLOCK, axis=1)
    prod = s * q.astype(np.float64)            # exact: 24-bit x 4-bit significands
    w = z + prod
    err = _two_sum_error(z, prod, w)
    if np.any(err != 0):
        raise ArithmeticError("zero + scale*q is not exact in fp64 for this matrix")
    return w[:, :cols] if cols < nb * BLOCK else w


def dequantize_f32(data: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """The correctly rounded f32 weights RN_f32(zero + scale*q), f32 [R, C]."""
    return dequantize_exact(data, rows, cols).astype(np.float32)


def pack_expert(gate: np.ndarray, up: np.ndarray, down: np.ndarray) -> np.ndarray:
    """One expert's bytes: [gate I x H][up I x H][down H x I] HFQ4 matrices."""
    return np.concatenate([quantize_matrix(gate), quantize_matrix(up), quantize_matrix(down)])


def expert_views(expert: np.ndarray, hidden: int, inter: int):
    """Split one expert's bytes into its three matrices' bytes."""
    mg = matrix_bytes(inter, hidden)
    md = matrix_bytes(hidden, inter)
    return expert[:mg], expert[mg:2 * mg], expert[2 * mg:2 * mg + md]


def dequantize_expert(expert: np.ndarray, hidden: int, inter: int):
    """(Wg [I,H], Wu [I,H], Wd [H,I]) exact f64 weights of one packed expert."""
    g, u, d = expert_views(expert, hidden, inter)
    return (dequantize_exact(g, inter, hidden), dequantize_exact(u, inter, hidden),
            dequantize_exact(d, hidden, inter))
