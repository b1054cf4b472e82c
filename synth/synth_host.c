/*
 * synth_host.c - host side of the seeded input generator (see synth_philox.h).
 *
 * Fills f32 arrays with the same bits that synth_dev.cu writes on the GPU.
 * Weight tensors are addressed by (layer, expert, matrix, row, col) so that
 * any single expert can be regenerated without the rest of the model.
 * Threads only split the index range; every element is a pure function of
 * its coordinates.
 */
#include <pthread.h>
#include <stdint.h>
#include <stddef.h>
#include "synth_philox.h"

typedef struct {
    float *out;
    uint64_t seed;
    uint32_t stream, a, b0;
    uint64_t per_b;    /* elements per b value */
    uint64_t begin, end;
    float factor;
} synth_job;

static void *synth_worker(void *arg)
{
    synth_job *j = (synth_job *)arg;
    for (uint64_t i = j->begin; i < j->end; ++i) {
        uint64_t bi = i / j->per_b, idx = i % j->per_b;
        synth_u32x4 r = synth_block(j->seed, j->stream, j->a, j->b0 + (uint32_t)bi, idx);
        j->out[i] = (float)synth_ih8_numerator(r) * j->factor;
    }
    return 0;
}

static void synth_run(float *out, uint64_t seed, uint32_t stream, uint32_t a, uint32_t b0,
                      uint64_t per_b, uint64_t total, double sigma, int n_threads)
{
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 64) n_threads = 64;
    if (total < 65536) n_threads = 1;
    synth_job jobs[64];
    pthread_t th[64];
    uint64_t chunk = (total + (uint64_t)n_threads - 1) / (uint64_t)n_threads;
    for (int t = 0; t < n_threads; ++t) {
        synth_job *j = &jobs[t];
        j->out = out; j->seed = seed; j->stream = stream; j->a = a; j->b0 = b0;
        j->per_b = per_b; j->factor = synth_normal_factor(sigma);
        j->begin = chunk * (uint64_t)t;
        j->end = j->begin + chunk > total ? total : j->begin + chunk;
        if (j->begin > total) j->begin = total;
    }
    if (n_threads == 1) { synth_worker(&jobs[0]); return; }
    for (int t = 0; t < n_threads; ++t) pthread_create(&th[t], 0, synth_worker, &jobs[t]);
    for (int t = 0; t < n_threads; ++t) pthread_join(th[t], 0);
}

/* out[e][r][c] for experts expert0..expert0+n_experts-1 of one matrix kind
 * (0 = gate, 1 = up, 2 = down, 3 = router) of one layer. */
void synth_weights_host(float *out, uint64_t seed, int layer, int expert0, int n_experts,
                        int matrix, int rows, int cols, double sigma, int n_threads)
{
    uint64_t per = (uint64_t)rows * (uint64_t)cols;
    /* b = expert*4 + matrix: consecutive experts are 4 apart, so run per expert. */
    for (int e = 0; e < n_experts; ++e)
        synth_run(out + per * (uint64_t)e, seed, SYNTH_STREAM_WEIGHT, (uint32_t)layer,
                  (uint32_t)((expert0 + e) * 4 + matrix), per, per, sigma, n_threads);
}

/* out[b][i] for b in b0..b0+nb-1, i < per_b: activations, logits, router rows. */
void synth_normal_host(float *out, uint64_t seed, uint32_t stream, uint32_t a, uint32_t b0,
                       int nb, uint64_t per_b, double sigma, int n_threads)
{
    synth_run(out, seed, stream, a, b0, per_b, per_b * (uint64_t)nb, sigma, n_threads);
}

/* 32-bit uniforms on (0,1) in double (host-only inputs such as Gumbel noise):
 * four per Philox block, element i takes word i%4 of block i/4. */
void synth_uniform_host(double *out, uint64_t seed, uint32_t stream, uint32_t a, uint32_t b,
                        uint64_t n)
{
    for (uint64_t i = 0; i < n; i += 4) {
        synth_u32x4 r = synth_block(seed, stream, a, b, i / 4);
        for (uint64_t w = 0; w < 4 && i + w < n; ++w) out[i + w] = synth_uniform01(r.v[w]);
    }
}

/* Logit-grade normals (synth_normal_fine), out[b][i] for b in b0..b0+nb-1. */
void synth_normal_fine_host(float *out, uint64_t seed, uint32_t stream, uint32_t a, uint32_t b0,
                            int nb, uint64_t per_b, double sigma)
{
    for (int b = 0; b < nb; ++b)
        for (uint64_t i = 0; i < per_b; ++i)
            out[(uint64_t)b * per_b + i] =
                synth_normal_fine(synth_block(seed, stream, a, b0 + (uint32_t)b, i), sigma);
}
