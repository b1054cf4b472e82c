/*
 * synth_philox.h - counter-based random numbers for the seeded synthetic
 * inputs (weights, activations, router logits).
 *
 * This header belongs to the input-generator module only.  It holds no step
 * of the MoE method: it turns (seed, stream, coordinates) into numbers, the
 * same bits on the host (synth_host.c) and on the GPU (synth_dev.cu).
 *
 * Generator: Philox4x32-10, from its published definition (J. K. Salmon,
 * M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel random numbers: as easy as
 * 1, 2, 3", SC'11, section 3.2): a 4x32-bit counter, a 2x32-bit key, ten
 * rounds of two 32x32->64 multiplies, with the key bumped by the Weyl
 * constants between rounds.
 *
 * Normal samples: Irwin-Hall sum of the eight 16-bit halves of one Philox
 * output.  With v_i uniform on {0..65535}, u_i = (v_i + 1/2) / 65536 is
 * uniform on (0,1) and sum(u_i) - 4 has variance 8/12, so
 *     z = (sum(v_i) - 262140) / 65536 * sqrt(12/8)
 * is a unit-variance, zero-mean approximation of N(0,1) with support
 * |z| < 4.9.  The integer numerator is below 2^19, so it is exact in f32, and
 * sigma*z is one correctly rounded f32 multiply of two exact f32 values:
 * identical on every IEEE machine.
 */
#ifndef SYNTH_PHILOX_H
#define SYNTH_PHILOX_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

/* Streams: which kind of tensor a number belongs to (folded into the key). */
enum {
    SYNTH_STREAM_WEIGHT = 1, /* expert weights: a = layer, b = expert*4 + matrix */
    SYNTH_STREAM_ACT = 2,    /* activations x:  a = layer (0), b = token */
    SYNTH_STREAM_LOGIT = 3,  /* router logits:  a = layer, b = token */
    SYNTH_STREAM_ROUTER = 4  /* router weights Wr: a = layer, b = expert */
};

/* Philox constants from the SC'11 paper (multipliers and Weyl key bumps). */
#define SYNTH_PHILOX_M0 0xD2511F53u
#define SYNTH_PHILOX_M1 0xCD9E8D57u
#define SYNTH_PHILOX_W0 0x9E3779B9u
#define SYNTH_PHILOX_W1 0xBB67AE85u

typedef struct { uint32_t v[4]; } synth_u32x4;

SYNTH_HD synth_u32x4 synth_philox4x32_10(synth_u32x4 ctr, uint32_t k0, uint32_t k1)
{
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = (uint64_t)SYNTH_PHILOX_M0 * (uint64_t)ctr.v[0];
        uint64_t p1 = (uint64_t)SYNTH_PHILOX_M1 * (uint64_t)ctr.v[2];
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        synth_u32x4 n;
        n.v[0] = hi1 ^ ctr.v[1] ^ k0;
        n.v[1] = lo1;
        n.v[2] = hi0 ^ ctr.v[3] ^ k1;
        n.v[3] = lo0;
        ctr = n;
        k0 += SYNTH_PHILOX_W0;
        k1 += SYNTH_PHILOX_W1;
    }
    return ctr;
}

/* One Philox block for element `idx` of tensor (stream, a, b) under `seed`. */
SYNTH_HD synth_u32x4 synth_block(uint64_t seed, uint32_t stream, uint32_t a,
                                 uint32_t b, uint64_t idx)
{
    synth_u32x4 c;
    c.v[0] = (uint32_t)idx;
    c.v[1] = (uint32_t)(idx >> 32);
    c.v[2] = a;
    c.v[3] = b;
    return synth_philox4x32_10(c, (uint32_t)seed, (uint32_t)(seed >> 32) ^ (stream * 0x85EBCA6Bu));
}

/* Integer numerator of the Irwin-Hall(8) normal: sum of 8 halves - 262140. */
SYNTH_HD int32_t synth_ih8_numerator(synth_u32x4 r)
{
    int32_t s = 0;
    for (int i = 0; i < 4; ++i) s += (int32_t)(r.v[i] & 0xFFFFu) + (int32_t)(r.v[i] >> 16);
    return s - 262140;
}

/* f32 factor sigma*sqrt(12/8)/65536, computed in double, rounded once. */
SYNTH_HD float synth_normal_factor(double sigma)
{
    return (float)(sigma * 1.2247448713915890491 / 65536.0);
}

/* Finer normal for router logits, where exact ties between the k-th and the
 * (k+1)-th largest logit must be rare: Irwin-Hall sum of the four 32-bit words,
 *     z = (sum(v_i) + 2 - 2^33) / 2^32 * sqrt(3),
 * evaluated in double (the numerator is an exact integer below 2^34) and
 * rounded once to f32 after the multiply by sigma.  Support |z| < 3.47. */
SYNTH_HD float synth_normal_fine(synth_u32x4 r, double sigma)
{
    int64_t n = (int64_t)r.v[0] + (int64_t)r.v[1] + (int64_t)r.v[2] + (int64_t)r.v[3] + 2
                - ((int64_t)1 << 33);
    double z = (double)n * (1.7320508075688772935 / 4294967296.0);
    return (float)(z * sigma);
}

/* Uniform on (0,1) with 32 random bits: (v + 1/2) / 2^32, in double. */
SYNTH_HD double synth_uniform01(uint32_t v)
{
    return ((double)v + 0.5) * (1.0 / 4294967296.0);
}

#endif /* SYNTH_PHILOX_H */
