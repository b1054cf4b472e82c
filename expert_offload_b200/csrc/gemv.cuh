// gemv.cuh - HFQ4 dot products in registers (hipfire thread, "HFQ quantisation
// format and GEMV": w = zero + scale * q per 256-weight block, so a block's
// dot product with x is zero * sum(x) + scale * sum(q * x)).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace hfq {

// 32 bytes of one block's payload (64 nibbles, elements 8i..8i+7 in word i)
// against 64 activations.  Nibble -> float: `prmt` puts the byte 0x80|q into
// bits 16..23 of 0x3F800000, giving exactly 1 + q/128 (even elements from
// w & 0x0F0F0F0F, odd ones from (w >> 4) & 0x0F0F0F0F); the offset 1 is
// removed afterwards with the lane's sums of x, and the factor 128 restored.
__device__ __forceinline__ float2 nib64_fma(const uint32_t (&w)[8], const float2 *xp)
{
    float2 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t lo = (w[i] & 0x0F0F0F0Fu) | 0x80808080u;
        const uint32_t hi = ((w[i] >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float2 f;
            f.x = __uint_as_float(__byte_perm(lo, 0x3F800000u, 0x7044u | (j << 8)));
            f.y = __uint_as_float(__byte_perm(hi, 0x3F800000u, 0x7044u | (j << 8)));
            // two scalar FMAs: measured faster on sm_100 than one packed f32x2 FMA here
            acc[j].x = fmaf(f.x, xp[4 * i + j].x, acc[j].x);
            acc[j].y = fmaf(f.y, xp[4 * i + j].y, acc[j].y);
        }
    }
    return make_float2((acc[0].x + acc[1].x) + (acc[2].x + acc[3].x),
                       (acc[0].y + acc[1].y) + (acc[2].y + acc[3].y));
}

__device__ __forceinline__ float finish_dot(float2 acc, float2 sx, float scale, float zero)
{
    const float sq = 128.0f * ((acc.x - sx.x) + (acc.y - sx.y));
    return fmaf(scale, sq, zero * (sx.x + sx.y));
}

__device__ __forceinline__ void lds_words(const uint8_t *p, uint32_t (&w)[8])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint2 v = *reinterpret_cast<const uint2 *>(p + 8 * i);
        w[2 * i] = v.x;
        w[2 * i + 1] = v.y;
    }
}

// 16 nibbles (one 8-byte chunk) against 16 values held as 8 float2.
__device__ __forceinline__ float2 nib16_fma(uint2 v, const float2 *hp)
{
    const uint32_t wv[2] = {v.x, v.y};
    float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t lo = (wv[i] & 0x0F0F0F0Fu) | 0x80808080u;
        const uint32_t hi = ((wv[i] >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float fx = __uint_as_float(__byte_perm(lo, 0x3F800000u, 0x7044u | (j << 8)));
            const float fy = __uint_as_float(__byte_perm(hi, 0x3F800000u, 0x7044u | (j << 8)));
            acc[j & 1].x = fmaf(fx, hp[4 * i + j].x, acc[j & 1].x);
            acc[j & 1].y = fmaf(fy, hp[4 * i + j].y, acc[j & 1].y);
        }
    }
    return make_float2(acc[0].x + acc[1].x, acc[0].y + acc[1].y);
}

// 16 nibbles (one 8-byte chunk) against 16 values held as 8 float2, added
// into acc (.x over the even elements, .y over the odd ones); same nibble
// decoding as nib64_fma.
__device__ __forceinline__ void nib16_fma_acc(uint2 v, const float2 *hp, float2 &acc)
{
    const uint32_t wv[2] = {v.x, v.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t lo = (wv[i] & 0x0F0F0F0Fu) | 0x80808080u;
        const uint32_t hi = ((wv[i] >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc.x = fmaf(__uint_as_float(__byte_perm(lo, 0x3F800000u, 0x7044u | (j << 8))), hp[4 * i + j].x, acc.x);
            acc.y = fmaf(__uint_as_float(__byte_perm(hi, 0x3F800000u, 0x7044u | (j << 8))), hp[4 * i + j].y, acc.y);
        }
    }
}

// acc + lo(w) * lo(x) + hi(w) * hi(x) over the bf16 halves of w and x: exact
// products, f32 accumulation (mixed-precision fma of sm_100).
__device__ __forceinline__ float fma2_bf16(uint32_t w, uint32_t x, float acc)
{
    asm("{ .reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
        "fma.rn.f32.bf16 %0, wh, xh, %0; }"
        : "+f"(acc)
        : "r"(w), "r"(x));
    return acc;
}

// One payload word (8 nibbles; element 2i in the low nibble of byte i) against
// its 8 activations, prepared by bf16_x_pairs.  A masked field N < 256 in the
// low byte of a 16-bit half is, read as bf16, exactly N * 2^-133 (subnormal
// below 128, exponent field 1 from 128 on: one linear scale), so plain masks
// turn nibbles into bf16 operands: w & 0x000F000F holds elements (0, 4),
// w & 0x00F000F0 elements (1, 5) times 16, and the same masks on w >> 8 give
// (2, 6) and (3, 7) times 16.  Returns acc + 2^-133 * sum_i q_i * X_i.
__device__ __forceinline__ float nib8_dot_bf16(uint32_t w, const uint32_t *X, float acc)
{
    const uint32_t t = w >> 8;
    acc = fma2_bf16(w & 0x000F000Fu, X[0], acc);
    acc = fma2_bf16(w & 0x00F000F0u, X[1], acc);
    acc = fma2_bf16(t & 0x000F000Fu, X[2], acc);
    acc = fma2_bf16(t & 0x00F000F0u, X[3], acc);
    return acc;
}

// 2^e as f32 for e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// v * 2^s, exact while the result stays normal, for s in [-252, 254]: two
// multiplications by representable powers of two.
__device__ __forceinline__ float scale2(float v, int s)
{
    const int s1 = s >> 1;
    return v * pow2f(s1) * pow2f(s - s1);
}

// The four bf16 pairs nib8_dot_bf16 takes for activations v[0..7] scaled by
// 2^s (exactly, for bf16-valued v away from overflow): (v0, v4), (v1, v5)/16,
// (v2, v6), (v3, v7)/16.
__device__ __forceinline__ void bf16_x_pairs(const float (&v)[8], int s, uint32_t *X)
{
    const int o[4][2] = {{0, 4}, {1, 5}, {2, 6}, {3, 7}};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int sp = (p & 1) ? s - 4 : s;
        const __nv_bfloat162 b = __floats2bfloat162_rn(scale2(v[o[p][0]], sp), scale2(v[o[p][1]], sp));
        X[p] = *reinterpret_cast<const uint32_t *>(&b);
    }
}

// Scale exponent for a piece of activations whose largest magnitude is m:
// m * 2^s lies in [2^99, 2^100), so scaled products q * v * 2^(s - 133) stay
// normal f32 for every v within 2^-92 of m, and no sum overflows.  The result
// is in [-28, 225].
__device__ __forceinline__ int bf16_piece_scale(float m)
{
    const int e = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    return 99 - ((e ? e : 1) - 127);
}

// Padded column of activation c in shared memory: 2 floats after every 64, so
// the lanes' 64-wide slices start on distinct bank pairs.  Keeps even columns
// even (8-byte aligned float2 access).
__device__ __forceinline__ int xpad(int c) { return c + 2 * (c >> 6); }

}  // namespace hfq
