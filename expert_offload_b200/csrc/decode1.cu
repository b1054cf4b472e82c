// decode1.cu - persistent decode kernel for ONE token: every MoE layer of a
// decode step in one cooperative launch, one CTA of eight warps per SM.
//
// hipfire thread, "HFQ quantisation format and GEMV": token decode is a GEMV
// over 136-byte blocks, bound by the bytes of the k selected experts.  With one
// token, a CTA's share of a layer is a fixed pattern: for each routed slot j,
// rows [c*I/G, (c+1)*I/G) of the expert's gate and up matrices and rows
// [c*H/G, (c+1)*H/G) of its down matrix (c = this CTA, G = CTAs).  Per layer:
//   1. the CTA routes the token (softmax top-k, renormalised; hipfire
//      offload explainer, opening section): the warp maxima bound the k-th
//      logit, the experts at or above the bound are ranked by unique keys
//      (topk.cuh).  Layer l's logits are read only after layer l-1 has
//      finished everywhere, or, with the router in the loop, computed from
//      x_l (each CTA a share, exchanged as tagged words).  Warp 0 then issues the 2k gate/up
//      bulk copies (1-D TMA, no multicast), lane j for slot j, into k fixed
//      shared-memory slots with one mbarrier for gate/up and one for down per
//      slot; warp j issues slot j's down copy once its gate/up bytes are in.  Experts
//      in host memory are read by the owning warp with 16-byte loads over PCIe
//      (hipfire offload explainer, "PCIe pass-through").  Warps 1..7 prepare
//      their activation registers meanwhile.
//   2. warp w computes the gate/up rows of slot w (and w + 8) as soon as that
//      slot has landed: nibbles decoded in registers, warp-shuffle sums,
//      h = silu(g) * u into an L2-resident buffer as 8-byte {value, tag}
//      words, the tag naming this launch and layer.
//   3. warp w polls its slot's h words until every tag is this layer's (one
//      64-bit access reads a value with its tag, so no fence or counter is
//      needed), takes its slot's down rows against the full h, times the
//      routing weight; the eight warps' sums are added in a fixed order, the
//      bf16 residual is applied, and the CTA's rows of the next layer input
//      are written as tagged words too.
//   4. the next layer starts once this CTA has read every row of its input
//      with the next layer's tag, i.e. once every CTA has finished this one
//      (no separate grid barrier; h and x are double-buffered by layer
//      parity, which that ordering makes safe).
// The expert address table of layer l+1 comes into shared memory (cp.async)
// while layer l runs.  Every wait is bounded (sync.cuh); on expiry the status
// word holds HFQ_ERR_TIMEOUT and every CTA winds down.
#include <algorithm>

#include "device.cuh"
#include "gemv.cuh"
#include "ptx.cuh"
#include "sync.cuh"
#include "topk.cuh"

namespace hfq {
namespace {

constexpr int kW = 8;                   // warps
constexpr int kThr = kW * 32;
constexpr int kMaxK = 16;               // routed slots, two per warp
constexpr int kMaxDRows = 16;           // down rows per CTA (one batched warp reduction)
constexpr int kGuRows = 4;              // gate/up rows per batched warp reduction
constexpr int kXLoads = 4;              // 16-byte input loads per thread (H <= 2048)
constexpr int kHLoads = 8;              // 16-byte h loads per lane and slot (I <= 1024)
constexpr int kStamps = 32;             // timeline stamps per layer
constexpr int kMaxRouterRows = 4;       // router rows per CTA: E <= 512 over >= 128 CTAs
static_assert(kThr == 256, "the router's summation order has 8 groups of 32 partial sums");
constexpr int kSmemOptin = 232448;      // 227 KB per CTA on sm_100

struct D1Args {
    const void *const *eptr[HFQ_MAX_STACK_LAYERS];
    const uint8_t *eloc[HFQ_MAX_STACK_LAYERS];
    const float *logits;      // [L][E], or null when the routing is given or computed
    const uint16_t *router;   // [L][E][H] bf16 router weights: logits = Wr x_l in the kernel, or null
    uint64_t *lbuf;           // [2][E] {f32 logit, tag} words (router): each CTA computes E/G logits
    float *logits_out;        // [L][E] the computed logits (router), or null
    const int32_t *idx_in;    // [k] given routing (single layer), or null
    const float *wts_in;
    const void *x0;           // [H] bf16
    uint16_t *x_out;          // [H] bf16 input of the layer after the last, or null
    uint64_t *xbuf;           // [2][H] {bf16 value, tag} words, ping-pong between layers (L > 1)
    uint64_t *h;              // [2][k][Ip] {f32 value, tag} words, ping-pong between layers
    float *y;                 // [L][H], or null
    uint16_t *y_bf16;         // [H] of the last layer, or null
    int32_t *idx_all;         // [L][k], or null
    float *wts_all;
    unsigned *ctl;            // control block (device.cuh)
    long long timeout_ns;
    unsigned long long *timeline;   // debug: [2][L][kStamps] %globaltimer stamps, or null
    int L, E, k, H, I;
    int extra_arrivals;       // test hook: nonzero makes the layer-1 input poll (one layer: the h poll)
                              // expect a tag nobody writes
    // shared-memory layout, bytes; a slot is [gate span][up span][down span]
    int slot_bytes, up_off, down_off;
    int xs_off, ptab_off, ltab_off, ysh_off, lsm_off, rsm_off, sh_off;
    int ltab_stride;
};

struct D1Shared {
    uint64_t gu_bar[kMaxK];           // gate + up span of slot j landed
    uint64_t d_bar[kMaxK];            // down span of slot j landed
    uint64_t r_bar;                   // this CTA's router rows of a layer landed (one phase per layer)
    int r_issued;                     // router row copies issued
    float rpart[kMaxRouterRows * kW];     // router: the warps' partial sums of each row
    const uint8_t *base[kMaxK];       // expert of slot j
    float w[kMaxK];                   // routing weight of slot j
    unsigned hostmask;                // slots whose expert is in host memory
    int abort;
    int last_cta;
    int armed;                        // layers whose slot barriers were armed
    alignas(16) uint64_t rkey[HFQ_MAX_EXPERTS];   // routing: every expert's key
    alignas(16) uint64_t rcand[8 * kMaxK];        // the k best of each group of 64
    uint64_t rsel[kMaxK];             // the k best, by slot
    uint32_t rwmax[kW];               // routing (k <= 8): each warp's largest key
    int rn;                           // routing (k <= 8): experts at or above the bound
};

// Exchange tag of layer l (< 64) in launch `epoch`: never 0 (a fresh or
// cleared buffer), and as f32 a signalling NaN, which no h value that another
// kernel leaves in the buffer is.  The epoch keeps 13 bits, so a word last
// written 8192 launches ago could carry this launch's tag.  That cannot
// happen while consecutive launches share the exchange layout (k, padded I,
// H, one layer or several): each launch then rewrites at every layer every
// word it reads, so an unwritten word holds this launch's layer l - 2 or a
// layer of one of the two launches before.  When the layout differs from the
// last launch's (the shape signature below), the first thing a launch does is
// zero both exchange buffers everywhere, behind one grid-wide counter.
__device__ __forceinline__ uint32_t xch_tag(uint32_t epoch, int l)
{
    return 0x7FA00000u | ((epoch & 0x1FFFu) << 7) | (uint32_t)(l + 1);
}

// Signature of the exchange layout: bit 31 set (0 means none), k, padded I,
// H, whether x is exchanged (several layers) and the logit exchange's E (0
// without the in-kernel router).
__host__ __device__ __forceinline__ uint32_t xch_signature(int k, int Ip, int H, int L, int E_router)
{
    return 0x80000000u | ((uint32_t)k << 26) | ((uint32_t)(Ip >> 8) << 23) | ((uint32_t)(H >> 7) << 18) |
           ((uint32_t)E_router << 1) | (L > 1 ? 1u : 0u);
}


__device__ __forceinline__ void st_tagged(uint64_t *p, float v, uint32_t tag)
{
    const uint64_t w = (uint64_t)__float_as_uint(v) | ((uint64_t)tag << 32);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

// Two tagged words (16-byte aligned); each 64-bit element is read atomically.
__device__ __forceinline__ void ld_tagged2(const uint64_t *p, uint64_t &a, uint64_t &b)
{
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

// Padded f32 column of activation c in shared memory: 4 floats after every 64,
// so the lanes' 64-wide slices start on distinct bank quads and stay 16-byte
// aligned (128-bit loads).
__device__ __forceinline__ int xp4(int c) { return c + 4 * (c >> 6); }

// One contiguous byte range of an expert, widened to 16-byte boundaries.
struct Span {
    uint32_t src;     // 16-aligned offset within the expert
    int len;          // bytes, a multiple of 16 (0 for no rows)
    int delta;        // offset of the first wanted byte within the span
};

__device__ __forceinline__ Span span_of(size_t off, size_t len)
{
    Span s;
    const size_t a16 = off & ~(size_t)15, e16 = (off + len + 15) & ~(size_t)15;
    s.src = (uint32_t)a16;
    s.len = len ? (int)(e16 - a16) : 0;
    s.delta = (int)(off - a16);
    return s;
}

template <bool kOn>
__device__ __forceinline__ void stamp(const D1Args &a, int l, int s)
{
    if (kOn && a.timeline && threadIdx.x == 0 && l < a.L) {
        const int slot = blockIdx.x == 0 ? 0 : (blockIdx.x == gridDim.x / 2 ? 1 : -1);
        if (slot >= 0) a.timeline[((size_t)slot * a.L + l) * kStamps + s] = globaltimer_ns();
    }
}

// Debug timeline, thread `who` of CTAs 0 and G/2: %globaltimer once `dep`
// (a value the stamp waits for) is available.
template <bool kOn>
__device__ __forceinline__ void stamp_dep(const D1Args &a, int l, int s, bool who, float dep)
{
    if (kOn && a.timeline && who && l < a.L) {
        const int slot = blockIdx.x == 0 ? 0 : (blockIdx.x == gridDim.x / 2 ? 1 : -1);
        if (slot >= 0) {
            uint64_t t;
            asm volatile("{ .reg .f32 d; mov.b32 d, %1; mov.u64 %0, %%globaltimer; }" : "=l"(t) : "f"(dep));
            a.timeline[((size_t)slot * a.L + l) * kStamps + s] = t;
        }
    }
}

// Warp-wide copy of `len` bytes (a multiple of 16) from host-mapped memory,
// four 16-byte loads in flight per lane.
__device__ void warp_copy_host(uint8_t *dst, const uint8_t *src, int len)
{
    const int lane = threadIdx.x & 31;
    for (int o = lane * 16; o < len; o += 32 * 16 * 4) {
        uint4 v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
            if (o + r * 512 < len) v[r] = ld_nc_v4(src + o + r * 512);
#pragma unroll
        for (int r = 0; r < 4; ++r)
            if (o + r * 512 < len) *reinterpret_cast<uint4 *>(dst + o + r * 512) = v[r];
    }
    __syncwarp();
}

// Warp 0: cp.async of layer l's expert addresses (and locations) into table
// buffer l & 1.
__device__ __forceinline__ void fetch_table(const D1Args &a, int l, uint8_t *ptab, uint8_t *ltab)
{
    const int lane = threadIdx.x & 31, b = l & 1;
    const uint8_t *src = reinterpret_cast<const uint8_t *>(a.eptr[l]);
    uint8_t *dst = ptab + (size_t)b * a.E * 8;
    for (int i = lane; i < a.E / 2; i += 32) cp_async16(dst + 16 * i, src + 16 * i);
    if (a.eloc[l])
        for (int i = lane; i < a.E / 16; i += 32)
            cp_async16(ltab + (size_t)b * a.ltab_stride + 16 * i, a.eloc[l] + 16 * i);
    cp_async_commit();
}

// kRouter: the launch computes the logits (a.router set); kSmallK: k <= kW
// routing; kFull: host-mapped experts, given routing, the debug timeline or
// the test hook are possible.
// One instantiation per combination keeps the code a launch runs small
// (instruction-cache misses were the largest stall reason): the router and
// rank routing out cut a step by 2 %, the host paths and stamps out by 4 %.
template <bool kRouter, bool kSmallK, bool kFull>
__global__ void __launch_bounds__(kThr, 1) decode1_kernel(const __grid_constant__ D1Args a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const int H = a.H, I = a.I, k = a.k, E = a.E;
    const int nbH = (H + kBlock - 1) / kBlock, nbI = (I + kBlock - 1) / kBlock;
    const int Hp = nbH * kBlock, Ip = nbI * kBlock;
    const int rowB_gu = nbH * kBlockBytes, rowB_d = nbI * kBlockBytes;
    const size_t mg = (size_t)I * rowB_gu;              // bytes of the gate (or up) matrix
    const int gu_lo = (int)((long long)c * I / G), gu_hi = (int)((long long)(c + 1) * I / G);
    const int d_lo = (int)((long long)c * H / G), d_hi = (int)((long long)(c + 1) * H / G);
    const int n_gu = gu_hi - gu_lo, n_d = d_hi - d_lo;
    const Span sg = span_of((size_t)gu_lo * rowB_gu, (size_t)n_gu * rowB_gu);
    const Span su = span_of(mg + (size_t)gu_lo * rowB_gu, (size_t)n_gu * rowB_gu);
    const Span sd = span_of(2 * mg + (size_t)d_lo * rowB_d, (size_t)n_d * rowB_d);

    uint8_t *slots = smem;
    float *xs = reinterpret_cast<float *>(smem + a.xs_off);          // [xp4(Hp)] f32
    uint8_t *ptab = smem + a.ptab_off;                                // [2][E] addresses
    uint8_t *ltab = smem + a.ltab_off;                                // [2][ltab_stride]
    float *ysh = reinterpret_cast<float *>(smem + a.ysh_off);        // [kW][kMaxDRows]
    float *lsm = reinterpret_cast<float *>(smem + a.lsm_off);        // [E] logits (router)
    uint16_t *rsm = reinterpret_cast<uint16_t *>(smem + a.rsm_off);  // [E/G rows][H] this CTA's Wr rows
    D1Shared &sh = *reinterpret_cast<D1Shared *>(smem + a.sh_off);
    const WaitCtx wc{a.ctl, a.timeout_ns, &sh.abort};
    const uint32_t epoch = *(volatile const unsigned *)(a.ctl + kCtlEpoch);
    const uint32_t sig = xch_signature(k, Ip, H, a.L, kRouter ? E : 0);
    const bool reset = *(volatile const unsigned *)(a.ctl + kCtlSig) != sig;
    // router: CTA c computes the logits of experts [r_lo, r_hi); their Wr rows
    // are one contiguous span, copied into rsm a layer ahead
    // given routing (a single layer's forward) only in the full instantiation
    const int32_t *const idx_in = kFull ? a.idx_in : nullptr;
    const bool route_in_kernel = kRouter && !idx_in;
    const int r_lo = (int)((long long)c * E / G), r_hi = (int)((long long)(c + 1) * E / G);
    const uint32_t r_len = route_in_kernel ? (uint32_t)((r_hi - r_lo) * H * 2) : 0u;
    auto issue_router = [&](int l) {       // thread 0
        if (r_len) {
            mbar_arrive_expect_tx(&sh.r_bar, r_len);
            bulk_g2s_hint(rsm, a.router + ((size_t)l * E + r_lo) * H, r_len, &sh.r_bar, l2_evict_first_policy());
        }
        sh.r_issued = l + 1;
    };

    if (tid == 0) {
        for (int j = 0; j < kMaxK; ++j) {
            mbar_init(&sh.gu_bar[j], 1);
            mbar_init(&sh.d_bar[j], 1);
        }
        mbar_init(&sh.r_bar, 1);
        sh.abort = 0;
        sh.armed = 0;
        sh.r_issued = 0;
        fence_mbar_init();
        if (route_in_kernel && a.L > 0) issue_router(0);
    }
    for (int i = H + tid; i < Hp; i += kThr) xs[xp4(i)] = 0.0f;   // padding, never rewritten
    if (warp == 0) fetch_table(a, 0, ptab, ltab);
    if (reset) {
        // another exchange layout ran last on these buffers: zero them (tag 0
        // matches no launch) and wait until every CTA has done its share
        const size_t nh = (size_t)2 * k * Ip, nx = a.L > 1 && a.xbuf ? (size_t)2 * H : 0;
        const size_t nl = kRouter ? (size_t)2 * E : 0;
        for (size_t i = (size_t)c * kThr + tid; i < nh + nx + nl; i += (size_t)G * kThr) {
            if (i < nh) a.h[i] = 0ull;
            else if (i < nh + nx) a.xbuf[i - nh] = 0ull;
            else a.lbuf[i - nh - nx] = 0ull;
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            atomicAdd(a.ctl + kCtlClear, 1u);
            if (!wait_counter_ge(wc, a.ctl + kCtlClear, (unsigned)G)) sh.abort = 1;
        }
    }
    // a reset that did not complete leaves the layers undone (nothing armed)
    const int n_layers = __syncthreads_or(sh.abort) ? 0 : a.L;

    for (int l = 0; l < n_layers; ++l) {
        stamp<kFull>(a, l, 0);
        const uint32_t par = l & 1;          // parity of this layer's slot-barrier phases
        // ---------------------------------------------- 1a. layer input -> xs
        if (l == 0) {
            // bf16 input, 8 values per 16-byte load
            for (int i = tid; i < H / 8; i += kThr) {
                const uint4 v = __ldcg(static_cast<const uint4 *>(a.x0) + i);
                float2 *dst = reinterpret_cast<float2 *>(xs + xp4(i * 8));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    dst[r] = make_float2(__uint_as_float(w4[r] << 16), __uint_as_float(w4[r] & 0xFFFF0000u));
            }
        } else {
            // poll the tagged words of x_l (pairs 2 i, 2 i + 1, i = tid + kThr m)
            // until every one carries layer l's tag: then every CTA has
            // finished layer l - 1 (the test hook expects a tag nobody writes)
            const uint64_t *xw = a.xbuf + (size_t)(l & 1) * H;
            const uint32_t tag = xch_tag(epoch, l) ^ (kFull && a.extra_arrivals && l == 1 ? 1u : 0u);
            unsigned pend = 0;
#pragma unroll
            for (int m = 0; m < kXLoads; ++m)
                if (2 * (tid + kThr * m) < H) pend |= 1u << m;
            uint64_t t0 = 0;
            for (int it = 0; pend; ++it) {
                uint64_t v[kXLoads][2];
#pragma unroll
                for (int m = 0; m < kXLoads; ++m)
                    if (pend >> m & 1u) ld_tagged2(xw + 2 * (tid + kThr * m), v[m][0], v[m][1]);
#pragma unroll
                for (int m = 0; m < kXLoads; ++m)
                    if ((pend >> m & 1u) && (uint32_t)(v[m][0] >> 32) == tag && (uint32_t)(v[m][1] >> 32) == tag) {
                        const int i = 2 * (tid + kThr * m);
                        *reinterpret_cast<float2 *>(xs + xp4(i)) =
                            make_float2(__uint_as_float((uint32_t)v[m][0] << 16), __uint_as_float((uint32_t)v[m][1] << 16));
                        pend &= ~(1u << m);
                    }
                if (it == 16) t0 = globaltimer_ns();
                if (pend && it > 16 && (it & 15) == 0) {
                    if (sh.abort || *(volatile unsigned *)a.ctl != 0u) {
                        sh.abort = 1;
                        break;
                    }
                    if (deadline_passed(t0, a.timeout_ns)) {
                        raise_timeout(wc);
                        break;
                    }
                }
            }
        }
        if (__syncthreads_or(sh.abort)) break;
        stamp<kFull>(a, l, 4);
        // ---------------------------------------------- 1a'. router (optional)
        // logits = Wr_l x_l for experts [r_lo, r_hi) from this CTA's rows in
        // rsm, in the summation order of moe_router_logits (same bits):
        // thread j (warp g = j / 32) sums the 8-column chunks 8 j + 2048 i in
        // order, each warp sums its 32 partials by a butterfly, and the 8 warp
        // sums are added as ((0+1)+(2+3))+((4+5)+(6+7)).  The logits go out
        // as tagged words, and every CTA polls all E of them into lsm.
        if (kRouter && route_in_kernel) {
            const uint32_t tag = xch_tag(epoch, l);
            const bool rok = __all_sync(0xffffffffu, !r_len || wait_mbar_phase(wc, &sh.r_bar, par));
            if (!rok) sh.abort = 1;
            const int nr = r_hi - r_lo;
            for (int r = 0; rok && r < nr; ++r) {
                const uint16_t *row = rsm + (size_t)r * H;
                float acc = 0.0f;
                for (int h0 = 8 * tid; h0 < H; h0 += 8 * kThr) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + h0);
                    const float4 xa = *reinterpret_cast<const float4 *>(xs + xp4(h0));
                    const float4 xb = *reinterpret_cast<const float4 *>(xs + xp4(h0) + 4);
                    acc = fmaf(xa.x, __uint_as_float(v.x << 16), acc);
                    acc = fmaf(xa.y, __uint_as_float(v.x & 0xFFFF0000u), acc);
                    acc = fmaf(xa.z, __uint_as_float(v.y << 16), acc);
                    acc = fmaf(xa.w, __uint_as_float(v.y & 0xFFFF0000u), acc);
                    acc = fmaf(xb.x, __uint_as_float(v.z << 16), acc);
                    acc = fmaf(xb.y, __uint_as_float(v.z & 0xFFFF0000u), acc);
                    acc = fmaf(xb.z, __uint_as_float(v.w << 16), acc);
                    acc = fmaf(xb.w, __uint_as_float(v.w & 0xFFFF0000u), acc);
                }
                acc = warp_sum(acc);
                if (lane == 0) sh.rpart[r * kW + warp] = acc;
            }
            __syncthreads();
            if (rok && tid < nr) {
                const float *q = sh.rpart + tid * kW;
                const float logit = ((q[0] + q[1]) + (q[2] + q[3])) + ((q[4] + q[5]) + (q[6] + q[7]));
                st_tagged(a.lbuf + (size_t)(l & 1) * E + r_lo + tid, logit, tag);
                // out now: without the fence the word reached the other CTAs
                // microseconds later while they polled
                __threadfence();
            }
            // polling starts once this CTA's logits are out (early pollers
            // slow the writers down)
            __syncthreads();
            // poll: thread tid reads logits tid and tid + kThr (E <= 512)
            const uint64_t *lw = a.lbuf + (size_t)(l & 1) * E;
            unsigned pend = (tid < E ? 1u : 0u) | (tid + kThr < E ? 2u : 0u);
            uint64_t t0 = 0;
            for (int it = 0; pend; ++it) {
                uint64_t v[2] = {0ull, 0ull};
#pragma unroll
                for (int m = 0; m < 2; ++m)
                    if (pend >> m & 1u)
                        asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v[m]) : "l"(lw + tid + kThr * m) : "memory");
#pragma unroll
                for (int m = 0; m < 2; ++m)
                    if ((pend >> m & 1u) && (uint32_t)(v[m] >> 32) == tag) {
                        lsm[tid + kThr * m] = __uint_as_float((uint32_t)v[m]);
                        pend &= ~(1u << m);
                    }
                if (it == 16) t0 = globaltimer_ns();
                if (pend && it > 16 && (it & 15) == 0) {
                    if (sh.abort || *(volatile unsigned *)a.ctl != 0u) {
                        sh.abort = 1;
                        break;
                    }
                    if (deadline_passed(t0, a.timeout_ns)) {
                        raise_timeout(wc);
                        break;
                    }
                }
            }
            if (__syncthreads_or(sh.abort)) break;
            stamp<kFull>(a, l, 31);
            // rsm is free again: the next layer's rows travel during this layer
            if (tid == 0 && l + 1 < n_layers) {
                fence_proxy_async_smem();
                issue_router(l + 1);
            }
            if (a.logits_out && c == 0)
                for (int e = tid; e < E; e += kThr) a.logits_out[(size_t)l * E + e] = lsm[e];
        }
        // ---------------------------------------------- 1b. route (all warps)
        int re = -1;
        float rw = 0.0f;
        if (!idx_in) {
            const float *row = kRouter ? lsm : a.logits + (size_t)l * E;
            auto logit_of = [&](int e) { return kRouter ? row[e] : __ldg(row + e); };
            if (kSmallK)
                cta_route_small_k<kThr>(logit_of, E, k, sh.rkey, sh.rwmax, &sh.rn, sh.rsel, re, rw);
            else
                cta_route_rank<kThr>(logit_of, E, k, sh.rkey, sh.rcand, sh.rsel, re, rw);
        }
        if (warp == 0) {
            // ------------------------------------------ 1c. issue copies
            cp_async_wait_all();
            __syncwarp();
            stamp_dep<kFull>(a, l, 29, lane == 0, 0.f);
            int e = re;
            float w = rw;
            if (idx_in && lane < k) { e = idx_in[lane]; w = a.wts_in[lane]; }
            stamp_dep<kFull>(a, l, 2, lane == 0, w);
            bool bad = lane < k && (unsigned)e >= (unsigned)E;
            const uint8_t *base = nullptr;
            int loc = 0;
            if (lane < k && !bad) {
                base = reinterpret_cast<const uint8_t *const *>(ptab + (size_t)par * E * 8)[e];
                bad = ((uintptr_t)base & 15u) != 0;         // bulk copies start on 16 bytes
            }
            if (__any_sync(0xffffffffu, bad)) {
                if (lane == 0) { atomicCAS(a.ctl, 0u, (unsigned)HFQ_ERR_ARG); sh.abort = 1; }
                __syncwarp();
            }
            if (lane < k && !bad) {
                loc = kFull && a.eloc[l] ? ltab[(size_t)par * a.ltab_stride + e] : 0;
                sh.base[lane] = base;
                sh.w[lane] = w;
                if (a.idx_all && c == 0) {
                    a.idx_all[(size_t)l * k + lane] = e;
                    a.wts_all[(size_t)l * k + lane] = w;
                }
            }
            const unsigned hm = __ballot_sync(0xffffffffu, lane < k && loc != 0);
            __syncwarp();
            stamp_dep<kFull>(a, l, 25, lane == 0, 0.f);
            if (!sh.abort) {
                // the slots were last read by the generic proxy (previous layer)
                fence_proxy_async_smem();
                if (lane < k) {
                    if (!loc) {
                        mbar_arrive_expect_tx(&sh.gu_bar[lane], (uint32_t)(sg.len + su.len));
                        mbar_arrive_expect_tx(&sh.d_bar[lane], (uint32_t)sd.len);
                    } else {
                        // host slot: its warp loads the bytes itself; keep the phases in step
                        mbar_arrive(&sh.gu_bar[lane]);
                        mbar_arrive(&sh.d_bar[lane]);
                    }
                }
                __syncwarp();
                stamp_dep<kFull>(a, l, 26, lane == 0, 0.f);
                if (lane < k && !loc) {
                    // expert bytes are read once per step: evict them first from L2
                    const uint64_t pol = l2_evict_first_policy();
                    uint8_t *slot = slots + (size_t)lane * a.slot_bytes;
                    if (sg.len) bulk_g2s_hint(slot, base + sg.src, (uint32_t)sg.len, &sh.gu_bar[lane], pol);
                    if (su.len) bulk_g2s_hint(slot + a.up_off, base + su.src, (uint32_t)su.len, &sh.gu_bar[lane], pol);
                }
                if (lane == 0) { sh.armed = l + 1; sh.hostmask = hm; }
                __syncwarp();
                stamp_dep<kFull>(a, l, 27, lane == 0, 0.f);
            }
            // next layer's table, after the copies: the proxy fence above must
            // not wait for it
            if (l + 1 < a.L) fetch_table(a, l + 1, ptab, ltab);
            stamp_dep<kFull>(a, l, 3, lane == 0, 0.f);
        }

        // ---------------------------------------------- 2. gate/up rows
        // lane: block pb of the row, quarter pq (64 weights, 32 payload bytes).
        // Its 64 activations stay in registers as scaled bf16 pairs (gemv.cuh,
        // nib8_dot_bf16); the 2 * kGuRows dots of a row group run side by side.
        const int pb = lane >> 2, pq = lane & 3;
        const bool has_piece = pb < nbH;
        uint32_t X[32];
        float sxp = 0.0f;                       // sum of the piece's activations
        int xs_exp = 0;                         // the piece's scale exponent
        {
            const float4 *xq = reinterpret_cast<const float4 *>(xs + xp4(has_piece ? pb * kBlock + pq * 64 : 0));
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float4 q = has_piece ? xq[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                sxp += (q.x + q.y) + (q.z + q.w);
                m = fmaxf(m, fmaxf(fmaxf(fabsf(q.x), fabsf(q.y)), fmaxf(fabsf(q.z), fabsf(q.w))));
            }
            xs_exp = bf16_piece_scale(m);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 q0 = has_piece ? xq[2 * i] : make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 q1 = has_piece ? xq[2 * i + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
                const float v[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                bf16_x_pairs(v, xs_exp, X + 4 * i);
            }
        }
        // warps 1..7 prepared their activations while warp 0 routed; the
        // routing's slot table is complete after this
        if (__syncthreads_or(sh.abort)) break;
        stamp<kFull>(a, l, 1);
        bool ok = true;
        for (int j = warp; j < k && ok; j += kW) {
            uint8_t *slot = slots + (size_t)j * a.slot_bytes;
            if (kFull && (sh.hostmask >> j & 1u)) {
                warp_copy_host(slot, sh.base[j] + sg.src, sg.len);
                warp_copy_host(slot + a.up_off, sh.base[j] + su.src, su.len);
            } else if (!wait_mbar_phase(wc, &sh.gu_bar[j], par)) {
                ok = false;
                break;
            } else if (lane == 0 && sd.len) {
                // the slot's down rows, now that its gate/up bytes are in; the
                // span was last read by the generic proxy (previous layer)
                fence_proxy_async_smem();
                bulk_g2s_hint(slot + a.down_off, sh.base[j] + sd.src, (uint32_t)sd.len, &sh.d_bar[j],
                              l2_evict_first_policy());
            }
            stamp_dep<kFull>(a, l, 5 + j, lane == 0 && (warp == 0 || warp == 7), 0.f);
            const uint8_t *g0 = slot + sg.delta, *u0 = slot + a.up_off + su.delta;
            for (int r0 = 0; r0 < n_gu; r0 += kGuRows) {
                constexpr int kD = 2 * kGuRows;      // the group's dots: gate rows, then up rows
                const uint8_t *pw[kD];
                float2 sz[kD];
                float acc[kD];
                bool live[kD];
#pragma unroll
                for (int i = 0; i < kD; ++i) {
                    const int r = r0 + (i % kGuRows);
                    live[i] = has_piece && r < n_gu;
                    const uint8_t *blk = (i < kGuRows ? g0 : u0) + (size_t)(live[i] ? r : 0) * rowB_gu +
                                         (has_piece ? pb : 0) * kBlockBytes;
                    sz[i] = live[i] ? *reinterpret_cast<const float2 *>(blk) : make_float2(0.f, 0.f);
                    pw[i] = blk + 8 + pq * 32;
                    acc[i] = 0.0f;
                }
#pragma unroll
                for (int wq = 0; wq < 4; ++wq) {      // 16 weights per step
#pragma unroll
                    for (int i = 0; i < kD; ++i) {
                        const uint2 w = live[i] ? *reinterpret_cast<const uint2 *>(pw[i] + 8 * wq) : make_uint2(0u, 0u);
                        acc[i] = nib8_dot_bf16(w.x, X + 8 * wq, acc[i]);
                        acc[i] = nib8_dot_bf16(w.y, X + 8 * wq + 4, acc[i]);
                    }
                }
                // partial = zero * sum(x) + scale * sum(q * x) over this lane's 64
                float v[kD];
#pragma unroll
                for (int i = 0; i < kD; ++i)
                    v[i] = live[i] ? fmaf(sz[i].x, scale2(acc[i], 133 - xs_exp), sz[i].y * sxp) : 0.f;
                // lane l: total of value (l >> 2) & 7, i.e. gate row (l >> 2) for
                // l < 16 and the matching up row 16 lanes higher
                const float g = warp_sum_many<2 * kGuRows>(v);
                const float u = __shfl_down_sync(0xffffffffu, g, 16);
                const int i = lane >> 2;
                if (lane < 16 && (lane & 3) == 0 && r0 + i < n_gu)
                    st_tagged(a.h + ((size_t)(l & 1) * k + j) * Ip + gu_lo + r0 + i, silu(g) * u, xch_tag(epoch, l));
            }
        }
        if (__syncthreads_or(!ok || sh.abort)) break;
        stamp<kFull>(a, l, 16);

        // ---------------------------------------------- 3. h exchange, down rows
        // down rows of host slots travel while other CTAs finish their h rows
        for (int j = warp; j < k; j += kW)
            if (kFull && (sh.hostmask >> j & 1u))
                warp_copy_host(slots + (size_t)j * a.slot_bytes + a.down_off, sh.base[j] + sd.src, sd.len);
        stamp<kFull>(a, l, 17);

        // this warp's weighted row sums, ysh[warp][ri], summed over its slots.
        // Lane: piece pc (64 values of h, one quarter of a block) of row rs of
        // each pass; P = Ip / 64 lanes per row, 32 / P rows per pass.
        const int P = nbI * 4, RP = 32 / P;
        const int pc = lane % P, rs = lane / P;
        if (lane < kMaxDRows) ysh[warp * kMaxDRows + lane] = 0.0f;
        for (int j = warp; j < k && ok; j += kW) {
            // h of slot j -> the slot's gate/up part, consumed by now (zeros past
            // I), then the lane's piece and its even/odd sums into registers
            const uint64_t *hj = a.h + ((size_t)(l & 1) * k + j) * Ip;
            float *hw = reinterpret_cast<float *>(slots + (size_t)j * a.slot_bytes);
            {
                // poll the slot's tagged h words (values 4 i .. 4 i + 3 of this
                // lane's float4 i) until each carries this layer's tag; every
                // load of a round is in flight before the tags are checked (the
                // test hook of a one-layer launch expects a tag nobody writes)
                const uint32_t tag = xch_tag(epoch, l) ^ (kFull && a.extra_arrivals && a.L == 1 ? 1u : 0u);
                float4 q4[kHLoads];
                unsigned pend = 0;
#pragma unroll
                for (int q = 0; q < kHLoads; ++q) {
                    const int i = lane + 32 * q;
                    q4[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (i < Ip / 4 && 4 * i < I) pend |= 1u << q;
                }
                uint64_t t0 = 0;
                for (int it = 0; __any_sync(0xffffffffu, pend != 0u); ++it) {
                    uint64_t v[kHLoads][4];
#pragma unroll
                    for (int q = 0; q < kHLoads; ++q)
                        if (pend >> q & 1u) {
                            const uint64_t *pp = hj + 4 * (lane + 32 * q);
                            ld_tagged2(pp, v[q][0], v[q][1]);
                            ld_tagged2(pp + 2, v[q][2], v[q][3]);
                        }
#pragma unroll
                    for (int q = 0; q < kHLoads; ++q)
                        if ((pend >> q & 1u) && (uint32_t)(v[q][0] >> 32) == tag && (uint32_t)(v[q][1] >> 32) == tag &&
                            (uint32_t)(v[q][2] >> 32) == tag && (uint32_t)(v[q][3] >> 32) == tag) {
                            q4[q] = make_float4(__uint_as_float((uint32_t)v[q][0]), __uint_as_float((uint32_t)v[q][1]),
                                                __uint_as_float((uint32_t)v[q][2]), __uint_as_float((uint32_t)v[q][3]));
                            pend &= ~(1u << q);
                        }
                    if (it == 16) t0 = globaltimer_ns();
                    if (it > 16 && (it & 15) == 0) {
                        int stop = sh.abort || *(volatile unsigned *)a.ctl != 0u;
                        if (!stop && deadline_passed(t0, a.timeout_ns)) {
                            if (lane == 0) raise_timeout(wc);
                            stop = 1;
                        }
                        if (__any_sync(0xffffffffu, stop)) {
                            if (lane == 0) sh.abort = 1;
                            ok = false;
                            break;
                        }
                    }
                }
                if (!ok) break;
                // piece c (64 values) at 68 * c floats: the lanes' pieces start on
                // distinct bank quads
#pragma unroll
                for (int q = 0; q < kHLoads; ++q) {
                    const int i = lane + 32 * q;
                    if (i < Ip / 4) reinterpret_cast<float4 *>(hw + (i >> 4) * 68)[i & 15] = q4[q];
                }
            }
            __syncwarp();
            float2 hr[32];
            float2 hs2 = make_float2(0.f, 0.f);
            {
                const float4 *hp = reinterpret_cast<const float4 *>(hw + pc * 68);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float4 q = hp[i];
                    hr[2 * i] = make_float2(q.x, q.y);
                    hr[2 * i + 1] = make_float2(q.z, q.w);
                    hs2.x += q.x + q.z;
                    hs2.y += q.y + q.w;
                }
            }
            __syncwarp();                              // the staging row is read; next slot may overwrite
            stamp_dep<kFull>(a, l, 21, lane == 0 && warp == 0, hs2.x);
            if (!(kFull && (sh.hostmask >> j & 1u)) && !wait_mbar_phase(wc, &sh.d_bar[j], par)) {
                ok = false;
                break;
            }
            stamp_dep<kFull>(a, l, 22, lane == 0 && warp == 0, 0.f);
            const uint8_t *d0 = slots + (size_t)j * a.slot_bytes + a.down_off + sd.delta +
                                (pc >> 2) * kBlockBytes;                 // this lane's block of each row
            const float wj = sh.w[j];
#pragma unroll 1
            for (int p0 = 0; p0 * RP < n_d; p0 += 4) {      // four passes side by side
                float v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int ri = (p0 + q) * RP + rs;
                    v[q] = 0.0f;
                    if (ri < n_d) {
                        const uint8_t *blk = d0 + (size_t)ri * rowB_d;
                        const float2 sz = *reinterpret_cast<const float2 *>(blk);
                        uint32_t wv[8];
                        lds_words(blk + 8 + (pc & 3) * 32, wv);
                        v[q] = finish_dot(nib64_fma(wv, hr), hs2, sz.x, sz.y);
                    }
                }
                // sum over the P lanes of each row (contiguous, P a power of two)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    for (int o = P >> 1; o > 0; o >>= 1) v[q] += __shfl_xor_sync(0xffffffffu, v[q], o);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int ri = (p0 + q) * RP + rs;
                    if (pc == 0 && ri < n_d) ysh[warp * kMaxDRows + ri] += wj * v[q];
                }
            }
        }
        stamp_dep<kFull>(a, l, 23, lane == 0 && warp == 0, ysh[warp * kMaxDRows]);
        if (__syncthreads_or(!ok || sh.abort)) break;
        stamp<kFull>(a, l, 19);

        // ---------------------------------------------- 4. combine, residual
        if (tid < n_d) {
            float y = 0.0f;
#pragma unroll
            for (int w = 0; w < kW; ++w) y += ysh[w * kMaxDRows + tid];
            const int r = d_lo + tid;
            const bool last = l == a.L - 1;
            if (a.y) a.y[(size_t)l * H + r] = y;
            if (a.y_bf16 && last) a.y_bf16[r] = float_to_bf16_bits(y);
            const uint16_t xb = float_to_bf16_bits(xs[xp4(r)] + y);
            if (last) {
                if (a.x_out) a.x_out[r] = xb;
            } else if (a.xbuf) {
                st_tagged(a.xbuf + (size_t)((l + 1) & 1) * H + r, __uint_as_float(xb), xch_tag(epoch, l + 1));
            }
        }
        stamp<kFull>(a, l, 20);
        // xs and ysh are read by the combine before the next layer rewrites them
        if (l + 1 < a.L && __syncthreads_or(sh.abort)) break;
    }

    // no copy may still be writing this CTA's shared memory when it exits
    if (tid == 0 && r_len && sh.r_issued > 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&sh.r_bar, (uint32_t)(sh.r_issued - 1) & 1u) && !deadline_passed(t0, a.timeout_ns)) {
        }
    }
    if (warp == 0) {
        cp_async_wait_all();
        const int armed = sh.armed;
        if (armed > 0 && lane < k) {
            const uint32_t p = (uint32_t)(armed - 1) & 1u;
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&sh.gu_bar[lane], p) && !deadline_passed(t0, a.timeout_ns)) {
            }
            t0 = globaltimer_ns();
            while (!mbar_try_wait(&sh.d_bar[lane], p) && !deadline_passed(t0, a.timeout_ns)) {
            }
        }
    }
    // the last CTA to finish clears the counters this launch used
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned old = atomicAdd(a.ctl + kCtlDone, 1u);
        sh.last_cta = old == (unsigned)G - 1;
    }
    __syncthreads();
    if (sh.last_cta) {
        __threadfence();
        if (tid == 0) {
            a.ctl[kCtlEpoch] = epoch + 1u;    // the next launch's tags differ
            a.ctl[kCtlSig] = sig;             // and it knows this launch's layout
        }
        if (*(volatile unsigned *)a.ctl == 0u) {
            for (int l = tid; l < a.L; l += kThr) {
                a.ctl[kCtlBar + l] = 0u;
                a.ctl[kCtlH + (size_t)l * kCtlHStride] = 0u;
            }
            __syncthreads();
            if (tid == 0) {
                __threadfence();
                a.ctl[kCtlClear] = 0u;
                a.ctl[kCtlDone] = 0u;
            }
        }
    }
}

inline size_t up16(size_t b) { return (b + 15) / 16 * 16; }

}  // namespace

// T = 1 decode through decode1_kernel.  HFQ_ERR_UNSUPPORTED (no message, no
// launch) for a shape or alignment this kernel does not take.
hfq_status decode1_launch(const hfq4_layer *layers, int L, const float *logits, const int32_t *idx_in,
                          const float *wts_in, const void *x0, bool x0_f32, int k, uint16_t *x_out,
                          uint16_t *xbuf, float *h, float *y, uint16_t *y_bf16, int32_t *idx_all,
                          float *wts_all, unsigned *ctl, long long timeout_ns, int extra_arrivals,
                          cudaStream_t s, const uint16_t *router, uint64_t *lbuf, float *logits_out)
{
    const int H = layers[0].hidden, I = layers[0].inter, E = layers[0].n_experts;
    const int G = sm_count();
    if (G <= 0) return fail(HFQ_ERR_CUDA, "no CUDA device");
    if (L < 1 || L > HFQ_MAX_STACK_LAYERS || k < 1 || k > kMaxK) return HFQ_ERR_UNSUPPORTED;
    if (expert_bytes(H, I) % 16) return HFQ_ERR_UNSUPPORTED;      // 16-byte aligned experts
    if (x0_f32) return HFQ_ERR_UNSUPPORTED;     // the bf16 operands need bf16-valued activations
    const int nbI_ = (I + kBlock - 1) / kBlock;
    if (nbI_ != 1 && nbI_ != 2 && nbI_ != 4) return HFQ_ERR_UNSUPPORTED;   // 4 nbI lanes per down row
    if (H > kBlock * 8 || H % 8 || I > kBlock * 4 || I % 16 || E > HFQ_MAX_EXPERTS || E % 16)
        return HFQ_ERR_UNSUPPORTED;
    if ((H + G - 1) / G > kMaxDRows || (L > 1 && !xbuf) || !aligned16(x0) || (xbuf && !aligned16(xbuf)))
        return HFQ_ERR_UNSUPPORTED;
    for (int l = 0; l < L; ++l)
        if (!aligned16(layers[l].expert_ptr) || (layers[l].expert_loc && !aligned16(layers[l].expert_loc)))
            return HFQ_ERR_UNSUPPORTED;

    D1Args a;
    memset(&a, 0, sizeof a);
    for (int l = 0; l < L; ++l) {
        a.eptr[l] = layers[l].expert_ptr;
        a.eloc[l] = layers[l].expert_loc;
    }
    if (router && (!lbuf || !aligned16(router) || H % 8 || (E + G - 1) / G > kMaxRouterRows))
        return HFQ_ERR_UNSUPPORTED;
    a.logits = logits; a.idx_in = idx_in; a.wts_in = wts_in; a.x0 = x0; a.x_out = x_out;
    a.router = router; a.lbuf = lbuf; a.logits_out = logits_out;
    a.xbuf = reinterpret_cast<uint64_t *>(xbuf); a.h = reinterpret_cast<uint64_t *>(h); a.y = y; a.y_bf16 = y_bf16; a.idx_all = idx_all; a.wts_all = wts_all;
    a.ctl = ctl; a.timeout_ns = timeout_ns; a.extra_arrivals = extra_arrivals;
    a.timeline = static_cast<unsigned long long *>(option_timeline());
    a.L = L; a.E = E; a.k = k; a.H = H; a.I = I;

    // shared-memory layout
    const int nbH = (H + kBlock - 1) / kBlock, nbI = (I + kBlock - 1) / kBlock;
    const size_t Hp = (size_t)nbH * kBlock;
    const size_t rowB_gu = (size_t)nbH * kBlockBytes, rowB_d = (size_t)nbI * kBlockBytes;
    const size_t gspan = up16((size_t)((I + G - 1) / G) * rowB_gu + 15);
    const size_t dspan = up16((size_t)((H + G - 1) / G) * rowB_d + 15);
    // the gate/up part of a slot also stages the slot's h in the down phase:
    // 4 nbI pieces of 64 floats, 68 apart
    const size_t gu_part = std::max(2 * gspan, up16((size_t)nbI * 4 * 68 * 4));
    const size_t slot = (gu_part + dspan + 127) / 128 * 128;
    size_t off = (size_t)k * slot;
    a.slot_bytes = (int)slot; a.up_off = (int)gspan; a.down_off = (int)gu_part;
    a.xs_off = (int)off;
    off += up16((Hp + 4 * (Hp >> 6)) * 4);
    a.ptab_off = (int)off;
    off += (size_t)2 * E * 8;
    a.ltab_stride = (int)up16((size_t)E);
    a.ltab_off = (int)off;
    off += (size_t)2 * a.ltab_stride;
    a.ysh_off = (int)off;
    off += (size_t)kW * kMaxDRows * 4;
    a.lsm_off = (int)off;
    off += router ? up16((size_t)E * 4) : 0;
    off = up16(off);
    a.rsm_off = (int)off;
    off += router ? up16((size_t)((E + G - 1) / G) * H * 2) : 0;
    a.sh_off = (int)up16(off);
    const size_t smem = (size_t)a.sh_off + sizeof(D1Shared);

    // the instantiation for this launch, and its shared-memory limit (set once)
    bool full = a.timeline != nullptr || idx_in != nullptr || extra_arrivals != 0;
    for (int l = 0; l < L; ++l) full = full || layers[l].expert_loc != nullptr;
    const int variant = (router ? 4 : 0) + (k <= kW ? 2 : 0) + (full ? 1 : 0);
    const void *const kernels[8] = {
        (const void *)decode1_kernel<false, false, false>, (const void *)decode1_kernel<false, false, true>,
        (const void *)decode1_kernel<false, true, false>,  (const void *)decode1_kernel<false, true, true>,
        (const void *)decode1_kernel<true, false, false>,  (const void *)decode1_kernel<true, false, true>,
        (const void *)decode1_kernel<true, true, false>,   (const void *)decode1_kernel<true, true, true>};
    const void *kernel = kernels[variant];
    static int dyn_limit[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (!dyn_limit[variant]) {
        int dev = 0, optin = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "decode kernel attributes: %s", cudaGetErrorString(e));
        int lim = optin - (int)fa.sharedSizeBytes;
        if (lim > kSmemOptin) lim = kSmemOptin;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "decode kernel attribute %d: %s", lim, cudaGetErrorString(e));
        dyn_limit[variant] = lim;
    }
    if (smem > (size_t)dyn_limit[variant]) return HFQ_ERR_UNSUPPORTED;
    int resident = 0;
    cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kernel, kThr, smem);
    if (oe != cudaSuccess || resident < 1) return HFQ_ERR_UNSUPPORTED;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kThr);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeCooperative;
    attrs[0].val.cooperative = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    void *params[] = {&a};
    cudaError_t e = cudaLaunchKernelExC(&cfg, kernel, params);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "decode kernel launch: %s", cudaGetErrorString(e));
    return HFQ_OK;
}

}  // namespace hfq
