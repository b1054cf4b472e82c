/*
 * synth_dev.cu - GPU side of the seeded input generator (see synth_philox.h).
 *
 * Writes the same f32 bits as synth_host.c, so that a whole model (tens of GB
 * of weights) can be generated where it is used, while a checker regenerates
 * any single expert on the host.  No step of the MoE method lives here.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include "synth_philox.h"

namespace {

__global__ void synth_normal_kernel(float *__restrict__ out, uint64_t seed, uint32_t stream,
                                    uint32_t a, uint32_t b0, uint32_t b_step, uint64_t per_b,
                                    uint64_t total, float factor)
{
    uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (; i < total; i += stride) {
        uint64_t bi = i / per_b, idx = i - bi * per_b;
        synth_u32x4 r = synth_block(seed, stream, a, b0 + (uint32_t)bi * b_step, idx);
        out[i] = __fmul_rn((float)synth_ih8_numerator(r), factor);
    }
}

int launch(float *out, uint64_t seed, uint32_t stream, uint32_t a, uint32_t b0, uint32_t b_step,
           uint64_t per_b, uint64_t total, double sigma, cudaStream_t s)
{
    if (total == 0) return 0;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (total + 255) / 256;
    uint64_t cap = (uint64_t)(sms > 0 ? sms : 1) * 16;
    if (blocks > cap) blocks = cap;
    synth_normal_kernel<<<(unsigned)blocks, 256, 0, s>>>(out, seed, stream, a, b0, b_step, per_b,
                                                         total, synth_normal_factor(sigma));
    return (int)cudaGetLastError();
}

}  // namespace

extern "C" {

/* out[e][r][c] for experts expert0.. of one matrix kind of one layer (device). */
int synth_weights_dev(float *out, uint64_t seed, int layer, int expert0, int n_experts,
                      int matrix, int rows, int cols, double sigma, void *stream)
{
    uint64_t per = (uint64_t)rows * (uint64_t)cols;
    return launch(out, seed, SYNTH_STREAM_WEIGHT, (uint32_t)layer,
                  (uint32_t)(expert0 * 4 + matrix), 4u, per, per * (uint64_t)n_experts, sigma,
                  (cudaStream_t)stream);
}

/* out[b][i], b in b0..b0+nb-1 (device). */
int synth_normal_dev(float *out, uint64_t seed, uint32_t stream_id, uint32_t a, uint32_t b0,
                     int nb, uint64_t per_b, double sigma, void *stream)
{
    return launch(out, seed, stream_id, a, b0, 1u, per_b, per_b * (uint64_t)nb, sigma,
                  (cudaStream_t)stream);
}

}  // extern "C"
