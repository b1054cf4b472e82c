// device.cuh - small device helpers shared by the kernels of libhfq4moe.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "common.h"

namespace hfq {

constexpr int kBlock = HFQ4_BLOCK;             // weights per HFQ4 block
constexpr int kBlockBytes = HFQ4_BLOCK_BYTES;  // bytes per HFQ4 block
constexpr int kPayload = 128;                  // nibble bytes per block

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b)
{
    return __uint_as_float(((uint32_t)b) << 16);
}

// Round-to-nearest-even f32 -> bf16 bits.
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

// Loads activation element i of a row stored as f32 or bf16.
__device__ __forceinline__ float load_act(const void *x, int dtype, size_t i)
{
    return dtype == HFQ_BF16 ? bf16_bits_to_float(static_cast<const uint16_t *>(x)[i])
                             : static_cast<const float *>(x)[i];
}

// Status word at the head of every workspace.
struct WsHeader {
    unsigned int status;      // 0 = ok, else an hfq_status (negative) stored as unsigned
    unsigned int pad[63];
};
constexpr size_t kWsHeader = sizeof(WsHeader);   // 256 bytes

inline cudaError_t launch_check() { return cudaGetLastError(); }

}  // namespace hfq
