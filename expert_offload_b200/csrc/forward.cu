// forward.cu - the routed-expert HFQ4 GEMV path (decode and speculative
// verify): gate/up GEMV with fused SiLU(gate)*up, then the down GEMV with the
// weighted combine fused into it.  Entry points hfq4_moe_forward and
// hfq4_moe_decode_stack.
//
// hipfire thread, "HFQ quantisation format and GEMV": decode is a GEMV over
// 136-byte blocks and bandwidth-bound.  Each warp owns output rows; lanes
// split a row's blocks into 8-byte chunks of 16 nibbles and reduce with warp
// shuffles; per block the dot product is factored as
//     sum_i (zero + scale*q_i) x_i = scale * sum_i q_i x_i + zero * sum_i x_i.
#include <cfloat>

#include "device.cuh"

namespace hfq {
namespace {

constexpr int kThreads = 256;            // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;
constexpr size_t kMaxDownSmem = 192 * 1024;   // k * ceil(I/256) <= 192 staged h vectors

// Dot product of one HFQ4 row (nb blocks) with a zero-padded f32 vector in
// shared memory.  Returns the full sum in every lane.
__device__ __forceinline__ float row_dot(const uint8_t *__restrict__ row, int nb,
                                         const float *__restrict__ xs)
{
    float acc = 0.0f;
    for (int c = threadIdx.x & 31; c < nb * 16; c += 32) {
        const int b = c >> 4, j = c & 15;
        const uint8_t *blk = row + (size_t)b * kBlockBytes;
        const float2 sz = *reinterpret_cast<const float2 *>(blk);       // scale, zero
        const uint2 nib = *reinterpret_cast<const uint2 *>(blk + 8 + j * 8);
        const float *xp = xs + b * kBlock + j * 16;
        float sq = 0.0f, sx = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float x0 = xp[i], x1 = xp[8 + i];
            sq = fmaf((float)((nib.x >> (4 * i)) & 15u), x0, sq);
            sq = fmaf((float)((nib.y >> (4 * i)) & 15u), x1, sq);
            sx += x0 + x1;
        }
        acc = fmaf(sz.x, sq, fmaf(sz.y, sx, acc));
    }
    return warp_sum(acc);
}

// An expert id from the caller outside [0, E): recorded as HFQ_ERR_ARG in the
// status word (read by hfq_workspace_status); the pair is skipped, so no
// address is formed from it.
__device__ __forceinline__ bool bad_expert(int e, int E, unsigned *status)
{
    if ((unsigned)e < (unsigned)E) return false;
    if (status) atomicCAS(status, 0u, (unsigned)HFQ_ERR_ARG);
    return true;
}

// Gate/up: CTA (pair p = t*k + j, row chunk).  h[p][r] = silu(g_r) * u_r.
__global__ void __launch_bounds__(kThreads)
gateup_kernel(const void *const *__restrict__ eptr, const void *__restrict__ x, int x_dtype,
              const int32_t *__restrict__ idx, int k, int E, int H, int I, float *__restrict__ h,
              unsigned *status)
{
    extern __shared__ float xs[];               // [nbH * 256]
    const int p = blockIdx.x, t = p / k;
    const int e = idx[p];
    if (bad_expert(e, E, threadIdx.x == 0 ? status : nullptr)) return;
    const int nbH = (H + kBlock - 1) / kBlock;
    for (int i = threadIdx.x; i < nbH * kBlock; i += kThreads)
        xs[i] = i < H ? load_act(x, x_dtype, (size_t)t * H + i) : 0.0f;
    __syncthreads();
    const uint8_t *base = static_cast<const uint8_t *>(eptr[e]);
    const size_t row_bytes = (size_t)nbH * kBlockBytes;
    const uint8_t *gate = base, *up = base + (size_t)I * row_bytes;
    const int warp = threadIdx.x >> 5;
    const int nbI = (I + kBlock - 1) / kBlock;
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int r = blockIdx.y * kRowsPerCta + warp * kRowsPerWarp + rr;
        if (r >= I) break;
        float g = row_dot(gate + r * row_bytes, nbH, xs);
        float u = row_dot(up + r * row_bytes, nbH, xs);
        if ((threadIdx.x & 31) == 0) h[(size_t)p * nbI * kBlock + r] = silu(g) * u;
    }
}

// Down + combine: CTA (token t, row chunk).  y[t][r] = sum_j w_j * Wd_ej[r] . h[t,j].
// With x_res != null also writes x_next[t][r] = bf16(x_res[t][r] + y[t][r]).
__global__ void __launch_bounds__(kThreads)
down_kernel(const void *const *__restrict__ eptr, const float *__restrict__ h,
            const int32_t *__restrict__ idx, const float *__restrict__ wts, int k, int E, int H, int I,
            float *__restrict__ y, uint16_t *__restrict__ y_bf16,
            const uint16_t *__restrict__ x_res, uint16_t *__restrict__ x_next, unsigned *status)
{
    extern __shared__ float hs[];               // [k][nbI * 256]
    const int t = blockIdx.x;
    // a token with an invalid expert id writes nothing (its gate/up pairs were
    // skipped too); the status word says why
    for (int j = 0; j < k; ++j)
        if (bad_expert(idx[(size_t)t * k + j], E, threadIdx.x == 0 ? status : nullptr)) return;
    const int nbI = (I + kBlock - 1) / kBlock, hl = nbI * kBlock;
    for (int i = threadIdx.x; i < k * hl; i += kThreads) {
        int j = i / hl, c = i - j * hl;
        hs[i] = c < I ? h[((size_t)t * k + j) * hl + c] : 0.0f;
    }
    __syncthreads();
    const int nbH = (H + kBlock - 1) / kBlock;
    const size_t gate_bytes = (size_t)I * nbH * kBlockBytes;
    const size_t row_bytes = (size_t)nbI * kBlockBytes;
    const int warp = threadIdx.x >> 5;
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int r = blockIdx.y * kRowsPerCta + warp * kRowsPerWarp + rr;
        if (r >= H) break;
        float acc = 0.0f;
        for (int j = 0; j < k; ++j) {
            const uint8_t *down =
                static_cast<const uint8_t *>(eptr[idx[(size_t)t * k + j]]) + 2 * gate_bytes;
            float o = row_dot(down + (size_t)r * row_bytes, nbI, hs + j * hl);
            acc = fmaf(wts[(size_t)t * k + j], o, acc);
        }
        if ((threadIdx.x & 31) == 0) {
            size_t o = (size_t)t * H + r;
            if (y) y[o] = acc;
            if (y_bf16) y_bf16[o] = float_to_bf16_bits(acc);
            if (x_next) x_next[o] = float_to_bf16_bits(bf16_bits_to_float(x_res[o]) + acc);
        }
    }
}

// Per-layer route for the decode stack (T <= 8 tokens, one warp each).
__global__ void stack_route_kernel(const float *__restrict__ logits, int T, int E, int k,
                                   int32_t *__restrict__ idx, float *__restrict__ wts,
                                   int32_t *__restrict__ idx_out, float *__restrict__ wts_out)
{
    const int t = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (t >= T) return;
    const float *l = logits + (size_t)t * E;
    // each lane keeps a bitmask of its selected experts (E <= 512 -> 16 per lane)
    uint32_t mine = 0;
    int sel[HFQ_MAX_TOPK];
    float sv[HFQ_MAX_TOPK];
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int s = 0, e = lane; e < E; ++s, e += 32) {
            if (mine >> s & 1u) continue;
            float v = l[e];
            if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        sel[j] = bi;
        sv[j] = bv;
        if ((bi & 31) == lane) mine |= 1u << (bi >> 5);
    }
    if (lane == 0) {
        float s = 0.0f, ex[HFQ_MAX_TOPK];
        for (int j = 0; j < k; ++j) { ex[j] = __expf(sv[j] - sv[0]); s += ex[j]; }
        for (int j = 0; j < k; ++j) {
            float w = ex[j] / s;
            idx[t * k + j] = sel[j];
            wts[t * k + j] = w;
            if (idx_out) { idx_out[t * k + j] = sel[j]; wts_out[t * k + j] = w; }
        }
    }
}

// h of T tokens x k slots in f32; for one token at least four times that:
// the one-token kernel exchanges h as 8-byte {value, tag} words in two
// buffers (layer parity).
size_t h_bytes(int T, int k, int I)
{
    size_t nbI = (I + kBlock - 1) / kBlock;
    return ((size_t)std::max(T, 4) * k * nbI * kBlock * sizeof(float) + 255) / 256 * 256;
}

// One of the two activation buffers of a decode stack: T x H bf16, and at
// least H 8-byte words (the one-token kernel's tagged residual stream uses
// both buffers as [2][H] {bf16 value, tag} words).
size_t act_bytes(int T, int H) { return (std::max((size_t)T * H * 2, (size_t)H * 8) + 255) / 256 * 256; }

int num_sms_fwd()
{
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

hfq_status check_ws(void *ws, size_t ws_bytes, size_t need)
{
    if (!ws || ws_bytes < need)
        return fail(HFQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    if ((uintptr_t)ws & 255) return fail(HFQ_ERR_ALIGN, "workspace must be 256-byte aligned");
    return HFQ_OK;
}

hfq_status launch_layer(const hfq4_layer &L, const void *x, int x_dtype, int T, const int32_t *idx,
                        const float *wts, int k, float *y, void *y_bf16, float *h,
                        const uint16_t *x_res, uint16_t *x_next, unsigned *status, cudaStream_t s)
{
    const int H = L.hidden, I = L.inter;
    const int nbH = (H + kBlock - 1) / kBlock, nbI = (I + kBlock - 1) / kBlock;
    const size_t smem_down = (size_t)k * nbI * kBlock * sizeof(float);
    if (smem_down > kMaxDownSmem)
        return fail(HFQ_ERR_UNSUPPORTED, "k * ceil(inter/256) = %d exceeds %d", k * nbI,
                    (int)(kMaxDownSmem / 1024));
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kMaxDownSmem);
        attr_set = true;
    }
    dim3 g1(T * k, (I + kRowsPerCta - 1) / kRowsPerCta);
    gateup_kernel<<<g1, kThreads, nbH * kBlock * sizeof(float), s>>>(
        L.expert_ptr, x, x_dtype, idx, k, L.n_experts, H, I, h, status);
    dim3 g2(T, (H + kRowsPerCta - 1) / kRowsPerCta);
    down_kernel<<<g2, kThreads, smem_down, s>>>(
        L.expert_ptr, h, idx, wts, k, L.n_experts, H, I, y, static_cast<uint16_t *>(y_bf16), x_res, x_next,
        status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "forward launch: %s", cudaGetErrorString(err));
    return HFQ_OK;
}

hfq_status check_layer(const hfq4_layer *layer, int k)
{
    if (!layer || !layer->expert_ptr) return fail(HFQ_ERR_ARG, "layer or expert_ptr is null");
    return check_shape(layer->hidden, layer->inter, layer->n_experts, k);
}

}  // namespace
}  // namespace hfq

namespace hfq {
static long long g_timeout_ns = 1000000000LL;   // 1 s per bounded wait
static int g_extra_arrivals = 0;
static void *g_timeline = nullptr;
void *option_timeline() { return g_timeline; }
long long option_wait_timeout_ns() { return g_timeout_ns; }
int option_take_extra_arrivals()
{
    int v = g_extra_arrivals;
    g_extra_arrivals = 0;
    return v;
}
}  // namespace hfq

using namespace hfq;

extern "C" {

hfq_status hfq_set_option(int option, long long value)
{
    switch (option) {
    case HFQ_OPT_WAIT_TIMEOUT_NS:
        if (value < 1000 || value > 60000000000LL)
            return fail(HFQ_ERR_ARG, "wait timeout %lld ns outside [1 us, 60 s]", value);
        g_timeout_ns = value;
        return ok();
    case HFQ_OPT_TEST_MISSING_ARRIVALS:
        if (value < 0 || value > 1024) return fail(HFQ_ERR_ARG, "bad value %lld", value);
        g_extra_arrivals = (int)value;
        return ok();
    case HFQ_OPT_TIMELINE_BUFFER:
        g_timeline = reinterpret_cast<void *>((uintptr_t)value);
        return ok();
    default:
        return fail(HFQ_ERR_ARG, "unknown option %d", option);
    }
}

size_t hfq4_moe_workspace_bytes(int T, int k, int hidden, int inter, int n_experts)
{
    if (T < 1 || k < 1 || hidden < 1 || inter < 1 || n_experts < 1) return 0;
    size_t b = stack_ctl_bytes() + h_bytes(T, k, inter);
    if (T > 8) b += tc_workspace_bytes(T, k, hidden, inter, n_experts);   // tensor-core path
    return b;
}

hfq_status hfq4_moe_forward(const hfq4_layer *layer, const void *x, hfq_dtype x_dtype, int T,
                            const int32_t *idx, const float *wts, int k, const int32_t *cnt,
                            const int32_t *off, const int32_t *perm, float *y, void *y_bf16,
                            int path, void *workspace, size_t ws_bytes, void *stream)
{
    hfq_status st = check_layer(layer, k);
    if (st) return st;
    if (!x || !idx || !wts || !y) return fail(HFQ_ERR_ARG, "hfq4_moe_forward: null pointer");
    if (T < 1 || T > 65536) return fail(HFQ_ERR_UNSUPPORTED, "T=%d not in [1, 65536]", T);
    if (x_dtype != HFQ_F32 && x_dtype != HFQ_BF16) return fail(HFQ_ERR_ARG, "bad x_dtype");
    if (path != HFQ_PATH_AUTO && path != HFQ_PATH_GEMV && path != HFQ_PATH_TC)
        return fail(HFQ_ERR_ARG, "unknown path %d", path);
    if (!aligned16(x) || !aligned16(y) || (y_bf16 && !aligned16(y_bf16)))
        return fail(HFQ_ERR_ALIGN, "x, y and y_bf16 must be 16-byte aligned");
    const bool grouped = cnt && off && perm;
    if ((cnt || off || perm) && !grouped) return fail(HFQ_ERR_ARG, "cnt, off and perm go together");
    size_t need = hfq4_moe_workspace_bytes(T, k, layer->hidden, layer->inter, layer->n_experts);
    if (path == HFQ_PATH_TC && T <= 8)
        need += tc_workspace_bytes(T, k, layer->hidden, layer->inter, layer->n_experts);
    if ((st = check_ws(workspace, ws_bytes, need))) return st;
    char *wsb = static_cast<char *>(workspace);
    float *h = reinterpret_cast<float *>(wsb + stack_ctl_bytes());
    cudaStream_t s = (cudaStream_t)stream;
    const bool use_tc = path == HFQ_PATH_TC ||
                        (path == HFQ_PATH_AUTO && T > 8 && grouped && tc_supported(layer->hidden, layer->inter));
    if (use_tc) {
        if (!grouped)
            return fail(HFQ_ERR_ARG, "the tensor-core path needs cnt, off and perm from moe_route");
        if (!tc_supported(layer->hidden, layer->inter))
            return fail(HFQ_ERR_UNSUPPORTED,
                        "tensor-core path: hidden and inter must be multiples of 128 with an even number of "
                        "256-weight blocks per row (hidden %d, inter %d)", layer->hidden, layer->inter);
        st = launch_tc(*layer, x, x_dtype == HFQ_F32, T, k, cnt, off, perm, wts, y,
                       static_cast<uint16_t *>(y_bf16), wsb + stack_ctl_bytes() + h_bytes(T, k, layer->inter),
                       static_cast<unsigned *>(workspace), option_wait_timeout_ns(), s);
    } else if (stack_supported(T, layer->hidden, layer->inter, k, num_sms_fwd())) {
        st = launch_stack(layer, 1, nullptr, idx, wts, x, x_dtype == HFQ_F32, T, k, nullptr,
                          nullptr, h, y, static_cast<uint16_t *>(y_bf16), nullptr, nullptr,
                          static_cast<unsigned *>(workspace), option_wait_timeout_ns(),
                          option_take_extra_arrivals(), s);
    } else {
        st = launch_layer(*layer, x, x_dtype, T, idx, wts, k, y, y_bf16, h, nullptr, nullptr,
                          static_cast<unsigned *>(workspace), s);
    }
    return st ? st : ok();
}

size_t hfq4_stack_workspace_bytes(int T, int k, int hidden, int inter, int n_experts)
{
    if (T < 1 || T > 8 || k < 1 || hidden < 1 || inter < 1 || n_experts < 1) return 0;
    // + the routed stack's logit exchange words [2][E], logits [T][E] and its
    // own pair of residual buffers (its per-layer fallback chains one-layer
    // stacks, which use the first pair)
    return stack_ctl_bytes() + h_bytes(T, k, inter) + 4 * act_bytes(T, hidden) +
           ((size_t)T * k * 8 + 255) / 256 * 256 + ((size_t)2 * n_experts * 8 + 255) / 256 * 256 +
           ((size_t)T * n_experts * 4 + 255) / 256 * 256;
}

int hfq4_stack_launches(int n_layers, int T, int k, int hidden, int inter)
{
    if (n_layers < 1 || n_layers > HFQ_MAX_STACK_LAYERS || T < 1 || T > 8 || k < 1) return 0;
    return stack_supported(T, hidden, inter, k, num_sms_fwd()) ? 1 : 3 * n_layers;
}

hfq_status hfq4_moe_decode_stack(const hfq4_layer *layers, int n_layers, const float *logits,
                                 int k, const void *x0, int T, void *x_out, float *y_all,
                                 int32_t *idx_all, float *wts_all, int path, void *workspace,
                                 size_t ws_bytes, void *stream)
{
    if (!layers || n_layers < 1 || n_layers > HFQ_MAX_STACK_LAYERS)
        return fail(HFQ_ERR_ARG, "n_layers=%d not in [1, %d]", n_layers, HFQ_MAX_STACK_LAYERS);
    hfq_status st;
    for (int l = 0; l < n_layers; ++l) {
        if ((st = check_layer(&layers[l], k))) return st;
        if (layers[l].hidden != layers[0].hidden || layers[l].inter != layers[0].inter ||
            layers[l].n_experts != layers[0].n_experts)
            return fail(HFQ_ERR_ARG, "layer %d has a different shape", l);
    }
    if (!logits || !x0 || !x_out) return fail(HFQ_ERR_ARG, "null pointer");
    if (T < 1 || T > 8) return fail(HFQ_ERR_UNSUPPORTED, "decode stack takes T in [1, 8], got %d", T);
    if ((idx_all == nullptr) != (wts_all == nullptr))
        return fail(HFQ_ERR_ARG, "idx_all and wts_all go together");
    if (path != HFQ_PATH_AUTO && path != HFQ_PATH_GEMV)
        return fail(HFQ_ERR_UNSUPPORTED, "decode stack runs the GEMV path only");
    if (!aligned16(x0) || !aligned16(x_out) || (y_all && !aligned16(y_all)))
        return fail(HFQ_ERR_ALIGN, "x0, x_out and y_all must be 16-byte aligned");
    const int H = layers[0].hidden, I = layers[0].inter, E = layers[0].n_experts;
    size_t need = hfq4_stack_workspace_bytes(T, k, H, I, E);
    if ((st = check_ws(workspace, ws_bytes, need))) return st;
    char *ws = static_cast<char *>(workspace) + stack_ctl_bytes();
    float *h = reinterpret_cast<float *>(ws);
    ws += h_bytes(T, k, I);
    uint16_t *xa = reinterpret_cast<uint16_t *>(ws);
    ws += act_bytes(T, H);
    uint16_t *xb = reinterpret_cast<uint16_t *>(ws);
    ws += act_bytes(T, H);
    int32_t *idx = reinterpret_cast<int32_t *>(ws);
    float *wts = reinterpret_cast<float *>(ws + (size_t)T * k * 4);
    cudaStream_t s = (cudaStream_t)stream;
    if (stack_supported(T, H, I, k, num_sms_fwd())) {
        st = launch_stack(layers, n_layers, logits, nullptr, nullptr, x0, false, T, k,
                          static_cast<uint16_t *>(x_out), xa, h, y_all, nullptr, idx_all, wts_all,
                          static_cast<unsigned *>(workspace), option_wait_timeout_ns(),
                          option_take_extra_arrivals(), s);
        return st ? st : ok();
    }
    const uint16_t *cur = static_cast<const uint16_t *>(x0);
    for (int l = 0; l < n_layers; ++l) {
        uint16_t *next = (l == n_layers - 1) ? static_cast<uint16_t *>(x_out) : (l & 1 ? xb : xa);
        stack_route_kernel<<<1, 32 * T, 0, s>>>(logits + (size_t)l * T * E, T, E, k, idx, wts,
                                                idx_all ? idx_all + (size_t)l * T * k : nullptr,
                                                wts_all ? wts_all + (size_t)l * T * k : nullptr);
        float *y = y_all ? y_all + (size_t)l * T * H : nullptr;
        st = launch_layer(layers[l], cur, HFQ_BF16, T, idx, wts, k, y, nullptr, h, cur, next,
                          static_cast<unsigned *>(workspace), s);
        if (st) return st;
        cur = next;
    }
    return ok();
}

hfq_status hfq4_moe_decode_stack_routed(const hfq4_layer *layers, int n_layers, const void *router,
                                        hfq_dtype router_dtype, int k, const void *x0, int T, void *x_out,
                                        float *y_all, int32_t *idx_all, float *wts_all, float *logits_all,
                                        void *workspace, size_t ws_bytes, void *stream)
{
    if (!layers || n_layers < 1 || n_layers > HFQ_MAX_STACK_LAYERS)
        return fail(HFQ_ERR_ARG, "n_layers=%d not in [1, %d]", n_layers, HFQ_MAX_STACK_LAYERS);
    hfq_status st;
    for (int l = 0; l < n_layers; ++l) {
        if ((st = check_layer(&layers[l], k))) return st;
        if (layers[l].hidden != layers[0].hidden || layers[l].inter != layers[0].inter ||
            layers[l].n_experts != layers[0].n_experts)
            return fail(HFQ_ERR_ARG, "layer %d has a different shape", l);
    }
    if (!router || !x0 || !x_out) return fail(HFQ_ERR_ARG, "null pointer");
    if (router_dtype != HFQ_F32 && router_dtype != HFQ_BF16) return fail(HFQ_ERR_ARG, "bad router dtype");
    if (T < 1 || T > 8) return fail(HFQ_ERR_UNSUPPORTED, "decode stack takes T in [1, 8], got %d", T);
    if ((idx_all == nullptr) != (wts_all == nullptr))
        return fail(HFQ_ERR_ARG, "idx_all and wts_all go together");
    if (!aligned16(x0) || !aligned16(x_out) || !aligned16(router) || (y_all && !aligned16(y_all)))
        return fail(HFQ_ERR_ALIGN, "x0, x_out, router and y_all must be 16-byte aligned");
    const int H = layers[0].hidden, I = layers[0].inter, E = layers[0].n_experts;
    size_t need = hfq4_stack_workspace_bytes(T, k, H, I, E);
    if ((st = check_ws(workspace, ws_bytes, need))) return st;
    char *ws = static_cast<char *>(workspace) + stack_ctl_bytes();
    float *h = reinterpret_cast<float *>(ws);
    ws += h_bytes(T, k, I);
    uint16_t *xa = reinterpret_cast<uint16_t *>(ws);        // with the next buffer: the x exchange
    ws += 2 * act_bytes(T, H);
    ws += ((size_t)T * k * 8 + 255) / 256 * 256;
    uint64_t *lbuf = reinterpret_cast<uint64_t *>(ws);
    ws += ((size_t)2 * E * 8 + 255) / 256 * 256;
    float *lscratch = reinterpret_cast<float *>(ws);
    ws += ((size_t)T * E * 4 + 255) / 256 * 256;
    uint16_t *ra = reinterpret_cast<uint16_t *>(ws);
    uint16_t *rb = reinterpret_cast<uint16_t *>(ws + act_bytes(T, H));
    cudaStream_t s = (cudaStream_t)stream;
    unsigned *ctl = static_cast<unsigned *>(workspace);
    const bool bf16 = router_dtype == HFQ_BF16;
    if (T == 1 && bf16 && stack_supported(T, H, I, k, num_sms_fwd())) {
        // the router fused into the one-token kernel
        st = decode1_launch(layers, n_layers, nullptr, nullptr, nullptr, x0, false, k,
                            static_cast<uint16_t *>(x_out), xa, h, y_all, nullptr, idx_all, wts_all, ctl,
                            option_wait_timeout_ns(), option_take_extra_arrivals(), s,
                            static_cast<const uint16_t *>(router), lbuf, logits_all);
        if (st != HFQ_ERR_UNSUPPORTED) return st ? st : ok();
    }
    // otherwise layer by layer: the router GEMV, then the layer on its logits
    const size_t rstride = (size_t)E * H * (bf16 ? 2 : 4);
    const void *cur = x0;
    for (int l = 0; l < n_layers; ++l) {
        float *lg = logits_all ? logits_all + (size_t)l * T * E : lscratch;
        if ((st = launch_router(cur, true, static_cast<const char *>(router) + l * rstride, bf16, T, E, H, lg, s)))
            return st;
        void *next = (l == n_layers - 1) ? x_out : (void *)(l & 1 ? rb : ra);
        st = hfq4_moe_decode_stack(&layers[l], 1, lg, k, cur, T, next, y_all ? y_all + (size_t)l * T * H : nullptr,
                                   idx_all ? idx_all + (size_t)l * T * k : nullptr,
                                   wts_all ? wts_all + (size_t)l * T * k : nullptr, HFQ_PATH_AUTO, workspace,
                                   ws_bytes, stream);
        if (st) return st;
        cur = next;
    }
    return ok();
}

hfq_status hfq_workspace_status(void *workspace, size_t ws_bytes, void *stream)
{
    if (!workspace && ws_bytes == 0) return noalloc_status((cudaStream_t)stream);
    if (!workspace || ws_bytes < kWsHeader) return fail(HFQ_ERR_ARG, "no workspace");
    unsigned int word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t err = cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "status read: %s", cudaGetErrorString(err));
    if (word != 0) {
        // the wound-down launch left its counters behind: clear the whole control block
        size_t n = ws_bytes < stack_ctl_bytes() ? ws_bytes : stack_ctl_bytes();
        cudaMemsetAsync(workspace, 0, n, s);
        cudaStreamSynchronize(s);
        const int st = (int)word;
        if (st == HFQ_ERR_ARG)
            return fail(HFQ_ERR_ARG, "a kernel found an invalid expert id or grouping (status %d)", st);
        return fail((hfq_status)st, "a device-side wait ran out (status %d)", st);
    }
    return ok();
}

}  // extern "C"
