// gemv.cuh - HFQ4 dot products in registers (hipfire thread, "HFQ quantisation
// format and GEMV": w = zero + scale * q per 256-weight block, so a block's
// dot product with x is zero * sum(x) + scale * sum(q * x)).
#pragma once

#include <cstdint>

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

// Padded column of activation c in shared memory: 2 floats after every 64, so
// the lanes' 64-wide slices start on distinct bank pairs.  Keeps even columns
// even (8-byte aligned float2 access).
__device__ __forceinline__ int xpad(int c) { return c + 2 * (c >> 6); }

}  // namespace hfq
