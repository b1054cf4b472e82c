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

// Sums each of V values (V a power of two, 2 <= V <= 32) over the 32 lanes
// with V - 1 + log2(32 / V) shuffles, in a chain five shuffles deep: at each
// of the first log2 V steps a lane keeps half of its values and adds its
// partner's copy of them.  Returns, in lane l, the total of value
// (l >> (5 - log2 V)) & (V - 1).  `a` is overwritten.
template <int V>
__device__ __forceinline__ float warp_sum_many(float (&a)[V])
{
    static_assert(V >= 2 && V <= 32 && (V & (V - 1)) == 0, "V: a power of two in [2, 32]");
    const int lane = threadIdx.x & 31;
    int m = 16;
#pragma unroll
    for (int n = V; n > 1; n >>= 1, m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = up ? a[i] : a[i + n / 2];
            const float keep = up ? a[i + n / 2] : a[i];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    float v = a[0];
#pragma unroll
    for (int mm = 32 / V / 2; mm > 0; mm >>= 1) v += __shfl_xor_sync(0xffffffffu, v, mm);
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

// Control block at the head of a persistent kernel's workspace, in 32-bit
// words: [0] status (the WsHeader word), [1] CTAs finished, [3..5] debug: the
// first bounded wait of the 2..8-token kernel that gave up (site, layer, item),
// [64 + l] grid barrier after layer l, [128 + 128 l] CTAs whose h rows of layer
// l are written.  Zero between launches: the last CTA of a launch clears what
// it used (a wait that gave up leaves its record until the status is read).
// [2] counts the CTAs of a one-token launch that have cleared its exchange
// buffers (only when the shape signature below changed).  After those
// kCtlWords words, [kCtlEpoch] counts the launches of the one-token kernel on
// this workspace (its exchange tags) and [kCtlSig] holds the shape signature
// of the last one (0 = none yet); neither is cleared between launches, and
// both are cleared with the control block after a device-side error.
constexpr int kCtlDone = 1, kCtlClear = 2, kCtlBar = 64, kCtlH = 128, kCtlHStride = 128;
constexpr size_t kCtlWords = kCtlH + (size_t)HFQ_MAX_STACK_LAYERS * kCtlHStride;
constexpr size_t kCtlEpoch = kCtlWords;
constexpr size_t kCtlSig = kCtlWords + 1;
constexpr size_t kCtlBytes = ((kCtlWords + 2) * 4 + 255) / 256 * 256;

inline cudaError_t launch_check() { return cudaGetLastError(); }

// Persistent decode kernel (stack.cu).
bool stack_supported(int T, int H, int I, int k, int G);
size_t stack_ctl_bytes();
size_t stack_ctl_clear_bytes();      // the leading control words a fresh launch needs at zero
hfq_status launch_stack(const hfq4_layer *layers, int L, const float *logits, const int32_t *idx_in,
                        const float *wts_in, const void *x0, bool x0_f32, int T, int k,
                        uint16_t *x_out, uint16_t *xbuf, float *h, float *y, uint16_t *y_bf16,
                        int32_t *idx_all, float *wts_all, unsigned *ctl, long long timeout_ns,
                        int extra_arrivals, cudaStream_t s);

// Persistent decode kernel for one token (decode1.cu); launch_stack hands T = 1
// to it when decode1_launch accepts the shape (else HFQ_ERR_UNSUPPORTED with no
// launch, and the general kernel runs).
// With `router` (bf16 [L][E][H]) the kernel computes each layer's logits
// from x_l itself (`lbuf`: [2][E] exchange words in the workspace;
// `logits_out`: optional [L][E] copy of them) instead of reading `logits`.
hfq_status decode1_launch(const hfq4_layer *layers, int L, const float *logits, const int32_t *idx_in,
                          const float *wts_in, const void *x0, bool x0_f32, int k, uint16_t *x_out,
                          uint16_t *xbuf, float *h, float *y, uint16_t *y_bf16, int32_t *idx_all,
                          float *wts_all, unsigned *ctl, long long timeout_ns, int extra_arrivals,
                          cudaStream_t s, const uint16_t *router = nullptr, uint64_t *lbuf = nullptr,
                          float *logits_out = nullptr);
// Persistent decode kernel for 2..8 tokens (verify.cu); launch_stack hands such
// batches to it when verify_launch accepts the shape (else HFQ_ERR_UNSUPPORTED
// with no launch, and the general kernel runs).
hfq_status verify_launch(const hfq4_layer *layers, int L, const float *logits, const int32_t *idx_in,
                         const float *wts_in, const void *x0, bool x0_f32, int T, int k, uint16_t *x_out,
                         uint16_t *xbuf, float *h, float *y, uint16_t *y_bf16, int32_t *idx_all,
                         float *wts_all, unsigned *ctl, long long timeout_ns, int extra_arrivals,
                         cudaStream_t s);
int sm_count();

// Router GEMV logits = x Wr^T for T tokens (pack_route.cu).
hfq_status launch_router(const void *x, bool x_bf16, const void *wr, bool wr_bf16, int T, int E, int H,
                         float *logits, cudaStream_t s);

// Tensor-core expert path (tc.cu).
size_t tc_workspace_bytes(int T, int k, int H, int I, int E);
bool tc_supported(int H, int I);
hfq_status launch_tc(const hfq4_layer &L, const void *x, bool x_f32, int T, int k, const int32_t *cnt,
                     const int32_t *off, const int32_t *perm, const float *wts, float *y,
                     uint16_t *y_bf16, void *ws, unsigned *status, long long timeout_ns,
                     cudaStream_t s);

// Status word of the allocation-free forward's array on the current device
// (noalloc.cu); hfq_workspace_status(NULL, 0, stream) returns it.
hfq_status noalloc_status(cudaStream_t s);

// Library options (hfq_set_option).
long long option_wait_timeout_ns();
int option_take_extra_arrivals();     // one-shot test hook
void *option_timeline();              // debug: device buffer for phase stamps, or null

}  // namespace hfq
