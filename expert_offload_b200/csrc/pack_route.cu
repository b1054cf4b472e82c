// pack_route.cu - device HFQ4 packer, dequantiser, top-k router with grouping
// by expert, and the read-bandwidth probe.
#include <cfloat>

#include "device.cuh"
#include "topk.cuh"

namespace hfq {
namespace {

// ------------------------------------------------------------------ packing
// One warp per 256-weight block (hipfire thread, "HFQ quantisation format and
// GEMV"): lane l owns elements 8l..8l+7, i.e. payload word l.  Every f32
// operation is an explicitly rounded intrinsic so that no multiply-add is
// contracted: the bytes equal the host packer's.
__global__ void pack_kernel(const float *__restrict__ gate, const float *__restrict__ up,
                            const float *__restrict__ down, int n_experts, int H, int I,
                            uint8_t *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const size_t nbH = (H + kBlock - 1) / kBlock, nbI = (I + kBlock - 1) / kBlock;
    const size_t gblocks = (size_t)I * nbH;                    // blocks of gate (and of up)
    const size_t dblocks = (size_t)H * nbI;
    const size_t per_expert = 2 * gblocks + dblocks;
    const size_t total = per_expert * n_experts;
    size_t gw = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const size_t nw = ((size_t)gridDim.x * blockDim.x) >> 5;
    for (; gw < total; gw += nw) {
        size_t e = gw / per_expert, r = gw - e * per_expert;
        const float *src;
        int cols;
        size_t row, blk;
        if (r < 2 * gblocks) {
            const float *m = r < gblocks ? gate : up;
            size_t rr = r < gblocks ? r : r - gblocks;
            row = rr / nbH;
            blk = rr - row * nbH;
            cols = H;
            src = m + ((size_t)e * I + row) * H;
        } else {
            size_t rr = r - 2 * gblocks;
            row = rr / nbI;
            blk = rr - row * nbI;
            cols = I;
            src = down + ((size_t)e * H + row) * I;
        }
        const int c0 = (int)blk * kBlock + lane * 8;
        float v[8];
        float mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            bool real = c0 + i < cols;
            v[i] = real ? src[c0 + i] : 0.0f;
            if (real) {
                mn = fminf(mn, v[i]);
                mx = fmaxf(mx, v[i]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const float scale = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        const float zero = mn;
        uint32_t word = 0;
        if (scale != 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (c0 + i < cols) {
                    float t = rintf(__fdiv_rn(__fsub_rn(v[i], zero), scale));
                    int q = (int)fminf(fmaxf(t, 0.0f), 15.0f);
                    word |= (uint32_t)q << (4 * i);
                }
            }
        }
        uint8_t *dst = out + gw * kBlockBytes;    // blocks are numbered in storage order
        if (lane == 0) {
            reinterpret_cast<float *>(dst)[0] = scale;
            reinterpret_cast<float *>(dst)[1] = zero;
        }
        reinterpret_cast<uint32_t *>(dst + 8)[lane] = word;
    }
}

// --------------------------------------------------------------- dequantise
__global__ void dequant_kernel(const uint8_t *__restrict__ blocks, int rows, int cols,
                               float *__restrict__ out)
{
    const size_t nb = (cols + kBlock - 1) / kBlock;
    const size_t total = (size_t)rows * cols;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        size_t r = i / cols, c = i - r * cols;
        const uint8_t *blk = blocks + (r * nb + c / kBlock) * kBlockBytes;
        int w = (int)(c % kBlock);
        float scale = reinterpret_cast<const float *>(blk)[0];
        float zero = reinterpret_cast<const float *>(blk)[1];
        int q = (blk[8 + (w >> 1)] >> ((w & 1) * 4)) & 15;
        out[i] = fmaf(scale, (float)q, zero);   // one rounding of zero + scale*q
    }
}

// ------------------------------------------------------------------- route
// One warp per token (hipfire offload explainer, opening section: top-8 of a
// layer's experts): the k largest logits, ties to the lower expert index, and
// their softmax renormalised over the selected k (topk.cuh).
constexpr int kRouteWarps = 4;

__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const float *__restrict__ logits, int T, int E, int k, int32_t *__restrict__ idx,
             float *__restrict__ wts)
{
    const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;                         // whole warps
    int e;
    float w;
    warp_route(logits + (size_t)t * E, E, k, e, w);
    if (lane < k) {
        idx[(size_t)t * k + lane] = e;
        wts[(size_t)t * k + lane] = w;
    }
}

// Grouping by expert, stable: three passes over chunks of kGroupChunk pairs.
constexpr int kGroupChunk = 512;

__global__ void group_hist_kernel(const int32_t *__restrict__ idx, int P, int E,
                                  int32_t *__restrict__ hist)
{
    __shared__ int h[HFQ_MAX_EXPERTS];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    int p = blockIdx.x * kGroupChunk + threadIdx.x;
    if (p < P) atomicAdd(&h[idx[p]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = h[e];
}

// Single CTA: per-expert totals, exclusive scan over experts, per-chunk bases.
__global__ void group_scan_kernel(int32_t *__restrict__ hist, int n_chunks, int E,
                                  int32_t *__restrict__ cnt, int32_t *__restrict__ off)
{
    __shared__ int tot[HFQ_MAX_EXPERTS + 1];
    constexpr int kU = 16;                      // chunk counts in flight per thread
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int s = 0;
        for (int c0 = 0; c0 < n_chunks; c0 += kU) {
            int v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) v[u] = c0 + u < n_chunks ? hist[(size_t)(c0 + u) * E + e] : 0;
#pragma unroll
            for (int u = 0; u < kU; ++u) s += v[u];
        }
        tot[e] = s;
        cnt[e] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) { int v = tot[e]; tot[e] = run; run += v; }
        tot[E] = run;
        for (int e = 0; e <= E; ++e) off[e] = tot[e];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int base = tot[e];
        for (int c0 = 0; c0 < n_chunks; c0 += kU) {
            int v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) v[u] = c0 + u < n_chunks ? hist[(size_t)(c0 + u) * E + e] : 0;
#pragma unroll
            for (int u = 0; u < kU; ++u)
                if (c0 + u < n_chunks) {
                    hist[(size_t)(c0 + u) * E + e] = base;
                    base += v[u];
                }
        }
    }
}

__global__ void group_scatter_kernel(const int32_t *__restrict__ idx, int P, int E,
                                     const int32_t *__restrict__ base, int32_t *__restrict__ perm)
{
    __shared__ int wcnt[kGroupChunk / 32][HFQ_MAX_EXPERTS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < (kGroupChunk / 32) * E; i += blockDim.x) wcnt[i / E][i % E] = 0;
    __syncthreads();
    const int p = blockIdx.x * kGroupChunk + tid;
    const int e = p < P ? idx[p] : -1;
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(mask & ((1u << lane) - 1u));
    if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(mask);
    __syncthreads();
    if (e >= 0) {
        int pos = base[(size_t)blockIdx.x * E + e] + rank;
        for (int w = 0; w < warp; ++w) pos += wcnt[w][e];
        perm[pos] = p;
    }
}

// -------------------------------------------------------------------- probe
__global__ void probe_read_kernel(const uint4 *__restrict__ src, size_t n16, int iters,
                                  unsigned long long *sink)
{
    uint32_t acc = 0;
    for (int it = 0; it < iters; ++it)
        for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
             i += (size_t)gridDim.x * blockDim.x) {
            uint4 v;
            asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(src + i));
            acc ^= v.x ^ v.y ^ v.z ^ v.w;
        }
    if (acc == 0x9E3779B9u) atomicAdd(sink, 1ull);   // keeps the loads live
}

int num_sms()
{
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

}  // namespace

// Router GEMV: logits[t][e] = sum_h x[t][h] * Wr[e][h] with f32 accumulation
// in a fixed order: 256 partial sums p_j (j = 32 g + lane, g = 0..7), p_j
// taking the 8-value chunks h0 = 8 j + 2048 i in turn (each chunk's products
// in order, fmaf); each group g of 32 partials summed by a butterfly over the
// lanes (xor 16, 8, 4, 2, 1); the 8 group sums added as
// ((q0 + q1) + (q2 + q3)) + ((q4 + q5) + (q6 + q7)).  The one-token
// persistent kernel's fused router takes the same steps with its 8 warps as
// the groups (same bits).  Here one warp per (token, expert) holds the 8
// groups' partials of its lane.
__global__ void router_kernel(const void *__restrict__ x, int x_bf16, const void *__restrict__ wr, int wr_bf16,
                              int T, int E, int H, float *__restrict__ logits)
{
    const int wg = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (wg >= T * E) return;
    const int t = wg / E, e = wg - t * E;
    float q[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        float acc = 0.0f;
        for (int h0 = 8 * (32 * g + lane); h0 < H; h0 += 2048) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const size_t xi = (size_t)t * H + h0 + i, wi = (size_t)e * H + h0 + i;
                const float xv = x_bf16 ? bf16_bits_to_float(static_cast<const uint16_t *>(x)[xi])
                                        : static_cast<const float *>(x)[xi];
                const float wv = wr_bf16 ? bf16_bits_to_float(static_cast<const uint16_t *>(wr)[wi])
                                         : static_cast<const float *>(wr)[wi];
                acc = fmaf(xv, wv, acc);
            }
        }
        q[g] = warp_sum(acc);
    }
    if (lane == 0) logits[(size_t)t * E + e] = ((q[0] + q[1]) + (q[2] + q[3])) + ((q[4] + q[5]) + (q[6] + q[7]));
}

hfq_status launch_router(const void *x, bool x_bf16, const void *wr, bool wr_bf16, int T, int E, int H,
                         float *logits, cudaStream_t s)
{
    const size_t warps = (size_t)T * E;
    router_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(x, x_bf16 ? 1 : 0, wr, wr_bf16 ? 1 : 0, T, E, H,
                                                              logits);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "router launch: %s", cudaGetErrorString(err));
    return HFQ_OK;
}

}  // namespace hfq

using namespace hfq;

extern "C" {

hfq_status moe_router_logits(const void *x, hfq_dtype x_dtype, int T, int hidden, const void *router,
                             hfq_dtype router_dtype, int n_experts, float *logits, void *stream)
{
    if (!x || !router || !logits) return fail(HFQ_ERR_ARG, "moe_router_logits: null pointer");
    if ((x_dtype != HFQ_F32 && x_dtype != HFQ_BF16) || (router_dtype != HFQ_F32 && router_dtype != HFQ_BF16))
        return fail(HFQ_ERR_ARG, "moe_router_logits: bad dtype");
    if (T < 1 || T > 65536 || hidden < 8 || hidden % 8 || n_experts < 1 || n_experts > HFQ_MAX_EXPERTS)
        return fail(HFQ_ERR_UNSUPPORTED, "moe_router_logits: T=%d hidden=%d n_experts=%d outside the limits",
                    T, hidden, n_experts);
    if (((uintptr_t)x & 15) || ((uintptr_t)router & 15))
        return fail(HFQ_ERR_ALIGN, "moe_router_logits: x and router must be 16-byte aligned");
    const hfq_status st = launch_router(x, x_dtype == HFQ_BF16, router, router_dtype == HFQ_BF16, T, n_experts,
                                        hidden, logits, (cudaStream_t)stream);
    return st ? st : ok();
}

hfq_status hfq4_pack_experts_device(const float *gate, const float *up, const float *down,
                                    int n_experts, int hidden, int inter, void *out,
                                    size_t out_bytes, void *stream)
{
    if (!gate || !up || !down || !out) return fail(HFQ_ERR_ARG, "hfq4_pack_experts_device: null");
    if (n_experts < 1 || hidden < 1 || inter < 1) return fail(HFQ_ERR_ARG, "bad sizes");
    size_t eb = expert_bytes(hidden, inter);
    if (out_bytes < eb * (size_t)n_experts)
        return fail(HFQ_ERR_ARG, "out_bytes=%zu < %zu needed", out_bytes, eb * (size_t)n_experts);
    if (((uintptr_t)out & 7) || ((uintptr_t)gate & 3) || ((uintptr_t)up & 3) || ((uintptr_t)down & 3))
        return fail(HFQ_ERR_ALIGN, "out must be 8-byte and inputs 4-byte aligned");
    size_t blocks = eb / kBlockBytes * (size_t)n_experts;       // one warp each
    size_t ctas = (blocks + 7) / 8;
    size_t cap = (size_t)num_sms() * 32;
    pack_kernel<<<(unsigned)(ctas < cap ? ctas : cap), 256, 0, (cudaStream_t)stream>>>(
        gate, up, down, n_experts, hidden, inter, static_cast<uint8_t *>(out));
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "pack launch: %s", cudaGetErrorString(err));
    return ok();
}

hfq_status hfq4_dequant(const void *blocks, int rows, int cols, float *out, void *stream)
{
    if (!blocks || !out || rows < 1 || cols < 1) return fail(HFQ_ERR_ARG, "hfq4_dequant: bad args");
    if ((uintptr_t)blocks & 7) return fail(HFQ_ERR_ALIGN, "blocks must be 8-byte aligned");
    size_t total = (size_t)rows * cols;
    size_t ctas = (total + 255) / 256, cap = (size_t)num_sms() * 16;
    dequant_kernel<<<(unsigned)(ctas < cap ? ctas : cap), 256, 0, (cudaStream_t)stream>>>(
        static_cast<const uint8_t *>(blocks), rows, cols, out);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "dequant launch: %s", cudaGetErrorString(err));
    return ok();
}

size_t hfq_route_workspace_bytes(int T, int E, int k)
{
    if (T < 1 || E < 1 || k < 1) return 0;
    size_t chunks = ((size_t)T * k + kGroupChunk - 1) / kGroupChunk;
    return chunks * (size_t)E * sizeof(int32_t);
}

hfq_status moe_route(const float *logits, int T, int E, int k, int32_t *idx, float *wts,
                     int32_t *cnt, int32_t *off, int32_t *perm, void *workspace, size_t ws_bytes,
                     void *stream)
{
    if (!logits || !idx || !wts) return fail(HFQ_ERR_ARG, "moe_route: null pointer");
    if (T < 1 || T > 65536) return fail(HFQ_ERR_UNSUPPORTED, "moe_route: T=%d not in [1, 65536]", T);
    if (E < 1 || E > HFQ_MAX_EXPERTS || k < 1 || k > HFQ_MAX_TOPK || k > E)
        return fail(HFQ_ERR_UNSUPPORTED, "moe_route: E=%d k=%d outside the limits", E, k);
    bool group = cnt || off || perm;
    if (group && !(cnt && off && perm))
        return fail(HFQ_ERR_ARG, "moe_route: cnt, off and perm go together");
    size_t need = hfq_route_workspace_bytes(T, E, k);
    if (group && (!workspace || ws_bytes < need))
        return fail(HFQ_ERR_WORKSPACE, "moe_route: grouping needs %zu bytes of workspace", need);
    cudaStream_t s = (cudaStream_t)stream;
    route_kernel<<<(T + kRouteWarps - 1) / kRouteWarps, kRouteWarps * 32, 0, s>>>(logits, T, E, k, idx, wts);
    if (group) {
        int P = T * k;
        int chunks = (P + kGroupChunk - 1) / kGroupChunk;
        int32_t *hist = static_cast<int32_t *>(workspace);
        group_hist_kernel<<<chunks, kGroupChunk, 0, s>>>(idx, P, E, hist);
        group_scan_kernel<<<1, 512, 0, s>>>(hist, chunks, E, cnt, off);
        group_scatter_kernel<<<chunks, kGroupChunk, 0, s>>>(idx, P, E, hist, perm);
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "route launch: %s", cudaGetErrorString(err));
    return ok();
}

hfq_status hfq_probe_read(const void *src, size_t bytes, int iters, uint64_t *sink, void *stream)
{
    if (!src || !sink || bytes < 16 || iters < 1) return fail(HFQ_ERR_ARG, "hfq_probe_read: bad args");
    if ((uintptr_t)src & 15) return fail(HFQ_ERR_ALIGN, "src must be 16-byte aligned");
    probe_read_kernel<<<num_sms() * 4, 512, 0, (cudaStream_t)stream>>>(
        static_cast<const uint4 *>(src), bytes / 16, iters,
        reinterpret_cast<unsigned long long *>(sink));
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "probe launch: %s", cudaGetErrorString(err));
    return ok();
}

}  // extern "C"
