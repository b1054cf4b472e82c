// decode1.cu - persistent decode kernel for ONE token: every MoE layer of a
// decode step in one cooperative launch, one CTA of eight warps per SM.
//
// hipfire thread, "HFQ quantisation format and GEMV": token decode is a GEMV
// over 136-byte blocks, bound by the bytes of the k selected experts.  With one
// token, a CTA's share of a layer is a fixed pattern: for each routed slot j,
// rows [c*I/G, (c+1)*I/G) of the expert's gate and up matrices and rows
// [c*H/G, (c+1)*H/G) of its down matrix (c = this CTA, G = CTAs).  Per layer:
//   1. warp 0 routes the token (softmax top-k, renormalised; hipfire offload
//      explainer, opening section), reading layer l's logits only after layer
//      l-1 has finished everywhere, and at once issues the 3k bulk copies
//      (1-D TMA, no multicast), lane j for slot j, into k fixed shared-memory
//      slots with one mbarrier for gate/up and one for down per slot.  Experts
//      in host memory are read by the owning warp with 16-byte loads over PCIe
//      (hipfire offload explainer, "PCIe pass-through").  Warps 1..7 load the
//      layer input meanwhile.
//   2. warp w computes the gate/up rows of slot w (and w + 8) as soon as that
//      slot has landed: nibbles decoded in registers, warp-shuffle sums,
//      h = silu(g) * u into an L2-resident buffer.
//   3. once a release counter shows every CTA's h rows written, warp w takes
//      its slot's down rows against the full h, times the routing weight; the
//      eight warps' sums are added in a fixed order, the bf16 residual is
//      applied, and the CTA's rows of the next layer input are written.
//   4. a grid-wide barrier ends the layer.
// The expert address table of layer l+1 comes into shared memory (cp.async)
// while layer l runs.  Every wait is bounded (sync.cuh); on expiry the status
// word holds HFQ_ERR_TIMEOUT and every CTA winds down.
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
constexpr int kMaxDRows = 16;           // down rows per CTA
constexpr int kMaxHChunks = 2;          // 16-value h chunks per lane (I <= 1024)
constexpr int kXLoads = 4;              // 16-byte input loads per thread (H <= 2048)
constexpr int kStamps = 32;             // timeline stamps per layer
constexpr int kSmemOptin = 232448;      // 227 KB per CTA on sm_100

struct D1Args {
    const void *const *eptr[HFQ_MAX_STACK_LAYERS];
    const uint8_t *eloc[HFQ_MAX_STACK_LAYERS];
    const float *logits;      // [L][E], or null when the routing is given
    const int32_t *idx_in;    // [k] given routing (single layer), or null
    const float *wts_in;
    const void *x0;           // [H] bf16 (f32 when x0_f32)
    uint16_t *x_out;          // [H] bf16 input of the layer after the last, or null
    uint16_t *xbuf;           // [2][H] bf16 ping-pong between layers (L > 1)
    float *h;                 // [k][Ip]
    float *y;                 // [L][H], or null
    uint16_t *y_bf16;         // [H] of the last layer, or null
    int32_t *idx_all;         // [L][k], or null
    float *wts_all;
    unsigned *ctl;            // control block (device.cuh)
    long long timeout_ns;
    unsigned long long *timeline;   // debug: [2][L][kStamps] %globaltimer stamps, or null
    int L, E, k, H, I;
    int x0_f32;
    int extra_arrivals;       // test hook: grid barriers wait for this many more CTAs
    // shared-memory layout, bytes; a slot is [gate span][up span][down span]
    int slot_bytes, up_off, down_off;
    int xs_off, ptab_off, ltab_off, ysh_off, sh_off;
    int ltab_stride;
};

struct D1Shared {
    uint64_t gu_bar[kMaxK];           // gate + up span of slot j landed
    uint64_t d_bar[kMaxK];            // down span of slot j landed
    const uint8_t *base[kMaxK];       // expert of slot j
    float w[kMaxK];                   // routing weight of slot j
    unsigned hostmask;                // slots whose expert is in host memory
    int abort;
    int last_cta;
    int armed;                        // layers whose slot barriers were armed
};

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

__device__ __forceinline__ void stamp(const D1Args &a, int l, int s)
{
    if (a.timeline && threadIdx.x == 0 && l < a.L) {
        const int slot = blockIdx.x == 0 ? 0 : (blockIdx.x == gridDim.x / 2 ? 1 : -1);
        if (slot >= 0) a.timeline[((size_t)slot * a.L + l) * kStamps + s] = globaltimer_ns();
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
    float *xs = reinterpret_cast<float *>(smem + a.xs_off);          // [xpad(Hp)] f32
    uint8_t *ptab = smem + a.ptab_off;                                // [2][E] addresses
    uint8_t *ltab = smem + a.ltab_off;                                // [2][ltab_stride]
    float *ysh = reinterpret_cast<float *>(smem + a.ysh_off);        // [kW][kMaxDRows]
    D1Shared &sh = *reinterpret_cast<D1Shared *>(smem + a.sh_off);
    const WaitCtx wc{a.ctl, a.timeout_ns, &sh.abort};

    if (tid == 0) {
        for (int j = 0; j < kMaxK; ++j) {
            mbar_init(&sh.gu_bar[j], 1);
            mbar_init(&sh.d_bar[j], 1);
        }
        sh.abort = 0;
        sh.armed = 0;
        fence_mbar_init();
    }
    for (int i = H + tid; i < Hp; i += kThr) xs[xpad(i)] = 0.0f;   // padding, never rewritten
    if (warp == 0) fetch_table(a, 0, ptab, ltab);
    __syncthreads();

    for (int l = 0; l < a.L; ++l) {
        stamp(a, l, 0);
        const uint32_t par = l & 1;          // parity of this layer's slot-barrier phases
        if (warp == 0) {
            // ------------------------------------------ 1a. route, issue copies
            cp_async_wait_all();
            __syncwarp();
            int e = -1;
            float w = 0.0f;
            if (a.idx_in) {
                if (lane < k) { e = a.idx_in[lane]; w = a.wts_in[lane]; }
            } else {
                warp_route(a.logits + (size_t)l * E, E, k, e, w);
            }
            if (l + 1 < a.L) fetch_table(a, l + 1, ptab, ltab);
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
                loc = a.eloc[l] ? ltab[(size_t)par * a.ltab_stride + e] : 0;
                sh.base[lane] = base;
                sh.w[lane] = w;
                if (a.idx_all && c == 0) {
                    a.idx_all[(size_t)l * k + lane] = e;
                    a.wts_all[(size_t)l * k + lane] = w;
                }
            }
            const unsigned hm = __ballot_sync(0xffffffffu, lane < k && loc != 0);
            __syncwarp();
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
                if (lane < k && !loc) {
                    uint8_t *slot = slots + (size_t)lane * a.slot_bytes;
                    if (sg.len) bulk_g2s(slot, base + sg.src, (uint32_t)sg.len, &sh.gu_bar[lane]);
                    if (su.len) bulk_g2s(slot + a.up_off, base + su.src, (uint32_t)su.len, &sh.gu_bar[lane]);
                    if (sd.len) bulk_g2s(slot + a.down_off, base + sd.src, (uint32_t)sd.len, &sh.d_bar[lane]);
                }
                if (lane == 0) { sh.armed = l + 1; sh.hostmask = hm; }
            }
        } else {
            // ------------------------------------------ 1b. layer input -> xs
            const void *xin = l == 0 ? a.x0 : (const void *)(a.xbuf + (size_t)(l & 1) * H);
            const bool f32 = l == 0 && a.x0_f32;
            const int per = f32 ? 4 : 8;                // values per 16-byte load
            const int nld = H / per;
            uint4 v[kXLoads];
#pragma unroll
            for (int q = 0; q < kXLoads; ++q) {
                const int i = tid - 32 + q * (kThr - 32);
                if (i < nld) v[q] = __ldcg(static_cast<const uint4 *>(xin) + i);
            }
#pragma unroll
            for (int q = 0; q < kXLoads; ++q) {
                const int i = tid - 32 + q * (kThr - 32);
                if (i >= nld) continue;
                float2 *dst = reinterpret_cast<float2 *>(xs + xpad(i * per));
                if (f32) {
                    dst[0] = make_float2(__uint_as_float(v[q].x), __uint_as_float(v[q].y));
                    dst[1] = make_float2(__uint_as_float(v[q].z), __uint_as_float(v[q].w));
                } else {
                    const uint32_t w4[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        dst[r] = make_float2(__uint_as_float(w4[r] << 16), __uint_as_float(w4[r] & 0xFFFF0000u));
                }
            }
        }
        if (__syncthreads_or(sh.abort)) break;
        stamp(a, l, 1);

        // ---------------------------------------------- 2. gate/up rows
        // lane: block pb of the row, quarter pq (64 weights, 32 payload bytes)
        const int pb = lane >> 2, pq = lane & 3;
        const bool has_piece = pb < nbH;
        float2 xr[32];
        float2 sx = make_float2(0.f, 0.f);
        {
            const float2 *xp = reinterpret_cast<const float2 *>(xs + xpad(has_piece ? pb * kBlock + pq * 64 : 0));
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                xr[i] = has_piece ? xp[i] : make_float2(0.f, 0.f);
                sx.x += xr[i].x;
                sx.y += xr[i].y;
            }
        }
        bool ok = true;
        for (int j = warp; j < k && ok; j += kW) {
            uint8_t *slot = slots + (size_t)j * a.slot_bytes;
            if (sh.hostmask >> j & 1u) {
                warp_copy_host(slot, sh.base[j] + sg.src, sg.len);
                warp_copy_host(slot + a.up_off, sh.base[j] + su.src, su.len);
            } else if (!wait_mbar_phase(wc, &sh.gu_bar[j], par)) {
                ok = false;
                break;
            }
            const uint8_t *g0 = slot + sg.delta, *u0 = slot + a.up_off + su.delta;
            for (int r = 0; r < n_gu; ++r) {
                float gd = 0.f, ud = 0.f;
                if (has_piece) {
                    const uint8_t *gb = g0 + (size_t)r * rowB_gu + pb * kBlockBytes;
                    const uint8_t *ub = u0 + (size_t)r * rowB_gu + pb * kBlockBytes;
                    const float2 gsz = *reinterpret_cast<const float2 *>(gb);
                    const float2 usz = *reinterpret_cast<const float2 *>(ub);
                    uint32_t gw[8], uw[8];
                    lds_words(gb + 8 + pq * 32, gw);
                    lds_words(ub + 8 + pq * 32, uw);
                    gd = finish_dot(nib64_fma(gw, xr), sx, gsz.x, gsz.y);
                    ud = finish_dot(nib64_fma(uw, xr), sx, usz.x, usz.y);
                }
                gd = warp_sum(gd);
                ud = warp_sum(ud);
                if (lane == 0) a.h[(size_t)j * Ip + gu_lo + r] = silu(gd) * ud;
            }
        }
        if (__syncthreads_or(!ok || sh.abort)) break;
        stamp(a, l, 16);

        // ---------------------------------------------- 3. h exchange, down rows
        unsigned *hcnt = a.ctl + kCtlH + (size_t)l * kCtlHStride;
        if (tid == 0) {
            __threadfence();
            red_release_gpu_add(hcnt, 1u);
        }
        // down rows of host slots travel while the counter fills
        for (int j = warp; j < k; j += kW)
            if (sh.hostmask >> j & 1u)
                warp_copy_host(slots + (size_t)j * a.slot_bytes + a.down_off, sh.base[j] + sd.src, sd.len);
        if (tid == 0) wait_counter_ge(wc, hcnt, (unsigned)G);
        if (__syncthreads_or(sh.abort)) break;
        stamp(a, l, 17);

        float acc[kMaxDRows];
#pragma unroll
        for (int ri = 0; ri < kMaxDRows; ++ri) acc[ri] = 0.0f;
        for (int j = warp; j < k && ok; j += kW) {
            // this lane's h chunks (16 values each) and their even/odd sums
            float2 hv[kMaxHChunks][8];
            float2 hsum[kMaxHChunks];
            const float *hj = a.h + (size_t)j * Ip;
#pragma unroll
            for (int m = 0; m < kMaxHChunks; ++m) {
                const int cc = lane + 32 * m;
                const bool okc = cc * 16 < I;
                hsum[m] = make_float2(0.f, 0.f);
                float4 q4[4];
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    q4[v] = okc ? __ldcg(reinterpret_cast<const float4 *>(hj + cc * 16) + v)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    hv[m][2 * v] = make_float2(q4[v].x, q4[v].y);
                    hv[m][2 * v + 1] = make_float2(q4[v].z, q4[v].w);
                    hsum[m].x += q4[v].x + q4[v].z;
                    hsum[m].y += q4[v].y + q4[v].w;
                }
            }
            if (!(sh.hostmask >> j & 1u) && !wait_mbar_phase(wc, &sh.d_bar[j], par)) {
                ok = false;
                break;
            }
            const uint8_t *d0 = slots + (size_t)j * a.slot_bytes + a.down_off + sd.delta;
            const float wj = sh.w[j];
#pragma unroll
            for (int ri = 0; ri < kMaxDRows; ++ri) {
                if (ri >= n_d) break;
                const uint8_t *row = d0 + (size_t)ri * rowB_d;
#pragma unroll
                for (int m = 0; m < kMaxHChunks; ++m) {
                    const int cc = lane + 32 * m;
                    if (cc * 16 >= I) continue;
                    const uint8_t *blk = row + (cc >> 4) * kBlockBytes;
                    const float2 sz = *reinterpret_cast<const float2 *>(blk);
                    const uint2 nv = *reinterpret_cast<const uint2 *>(blk + 8 + (cc & 15) * 8);
                    const float part = finish_dot(nib16_fma(nv, hv[m]), hsum[m], sz.x, sz.y);
                    acc[ri] = fmaf(wj, part, acc[ri]);
                }
            }
        }
#pragma unroll
        for (int ri = 0; ri < kMaxDRows; ++ri) {
            if (ri >= n_d) break;
            const float v = warp_sum(acc[ri]);
            if (lane == 0) ysh[warp * kMaxDRows + ri] = v;
        }
        if (__syncthreads_or(!ok || sh.abort)) break;
        stamp(a, l, 19);

        // ---------------------------------------------- 4. combine, residual
        if (tid < n_d) {
            float y = 0.0f;
#pragma unroll
            for (int w = 0; w < kW; ++w) y += ysh[w * kMaxDRows + tid];
            const int r = d_lo + tid;
            const bool last = l == a.L - 1;
            if (a.y) a.y[(size_t)l * H + r] = y;
            if (a.y_bf16 && last) a.y_bf16[r] = float_to_bf16_bits(y);
            uint16_t *xo = last ? a.x_out : (a.xbuf ? a.xbuf + (size_t)((l + 1) & 1) * H : nullptr);
            if (xo) xo[r] = float_to_bf16_bits(xs[xpad(r)] + y);
        }
        stamp(a, l, 20);
        if (l + 1 < a.L) {
            __syncthreads();
            if (tid == 0) {
                unsigned *bar = a.ctl + kCtlBar + l;
                __threadfence();
                red_release_gpu_add(bar, 1u);
                wait_counter_ge(wc, bar, (unsigned)(G + a.extra_arrivals));
            }
            if (__syncthreads_or(sh.abort)) break;
        }
    }

    // no copy may still be writing this CTA's shared memory when it exits
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
        if (*(volatile unsigned *)a.ctl == 0u) {
            for (int l = tid; l < a.L; l += kThr) {
                a.ctl[kCtlBar + l] = 0u;
                a.ctl[kCtlH + (size_t)l * kCtlHStride] = 0u;
            }
            __syncthreads();
            if (tid == 0) {
                __threadfence();
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
                          cudaStream_t s)
{
    const int H = layers[0].hidden, I = layers[0].inter, E = layers[0].n_experts;
    const int G = sm_count();
    if (L < 1 || L > HFQ_MAX_STACK_LAYERS || k < 1 || k > kMaxK) return HFQ_ERR_UNSUPPORTED;
    if (expert_bytes(H, I) % 16) return HFQ_ERR_UNSUPPORTED;      // 16-byte aligned experts
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
    a.logits = logits; a.idx_in = idx_in; a.wts_in = wts_in; a.x0 = x0; a.x_out = x_out;
    a.xbuf = xbuf; a.h = h; a.y = y; a.y_bf16 = y_bf16; a.idx_all = idx_all; a.wts_all = wts_all;
    a.ctl = ctl; a.timeout_ns = timeout_ns; a.extra_arrivals = extra_arrivals;
    a.timeline = static_cast<unsigned long long *>(option_timeline());
    a.L = L; a.E = E; a.k = k; a.H = H; a.I = I; a.x0_f32 = x0_f32 ? 1 : 0;

    // shared-memory layout
    const int nbH = (H + kBlock - 1) / kBlock, nbI = (I + kBlock - 1) / kBlock;
    const size_t Hp = (size_t)nbH * kBlock;
    const size_t rowB_gu = (size_t)nbH * kBlockBytes, rowB_d = (size_t)nbI * kBlockBytes;
    const size_t gspan = up16((size_t)((I + G - 1) / G) * rowB_gu + 15);
    const size_t dspan = up16((size_t)((H + G - 1) / G) * rowB_d + 15);
    const size_t slot = (2 * gspan + dspan + 127) / 128 * 128;
    size_t off = (size_t)k * slot;
    a.slot_bytes = (int)slot; a.up_off = (int)gspan; a.down_off = (int)(2 * gspan);
    a.xs_off = (int)off;
    off += up16((Hp + 2 * (Hp >> 6)) * 4);
    a.ptab_off = (int)off;
    off += (size_t)2 * E * 8;
    a.ltab_stride = (int)up16((size_t)E);
    a.ltab_off = (int)off;
    off += (size_t)2 * a.ltab_stride;
    a.ysh_off = (int)off;
    off += (size_t)kW * kMaxDRows * 4;
    a.sh_off = (int)up16(off);
    const size_t smem = (size_t)a.sh_off + sizeof(D1Shared);

    static int dyn_limit = 0;
    if (!dyn_limit) {
        int dev = 0, optin = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, decode1_kernel);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "decode kernel attributes: %s", cudaGetErrorString(e));
        int lim = optin - (int)fa.sharedSizeBytes;
        if (lim > kSmemOptin) lim = kSmemOptin;
        e = cudaFuncSetAttribute(decode1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "decode kernel attribute %d: %s", lim, cudaGetErrorString(e));
        dyn_limit = lim;
    }
    if (smem > (size_t)dyn_limit) return HFQ_ERR_UNSUPPORTED;
    int resident = 0;
    cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, decode1_kernel, kThr, smem);
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
    cudaError_t e = cudaLaunchKernelExC(&cfg, (const void *)decode1_kernel, params);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "decode kernel launch: %s", cudaGetErrorString(e));
    return HFQ_OK;
}

}  // namespace hfq
