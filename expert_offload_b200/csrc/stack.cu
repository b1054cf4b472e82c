// stack.cu - persistent decode kernel: every MoE layer of a decode step (or a
// single layer) in ONE cooperative launch, one CTA per SM.
//
// Per layer, every CTA:
//   1. routes the T tokens itself (warp per token: softmax top-k, renormalised,
//      hipfire offload explainer, opening section), reading layer l's logits
//      only after layer l-1 has finished everywhere;
//   2. lets its producer warp stream this CTA's share of every selected
//      expert's bytes into a shared-memory ring: rows [c*I/G, (c+1)*I/G) of
//      each expert's gate and up matrices, and rows [c*H/G, (c+1)*H/G) of each
//      expert's down matrix, with 1-D bulk copies (TMA, no multicast) from HBM
//      or plain 16-byte loads from host-mapped experts (hipfire explainer,
//      "PCIe pass-through"), in the order GU(0) GU(1) D(0) GU(2) D(1) ...;
//   3. has its consumer warps decode the nibbles in registers (hipfire thread,
//      "HFQ quantisation format and GEMV") and reduce with warp shuffles:
//      gate/up rows give h = silu(g)*u, written to an L2-resident buffer and
//      announced per expert with a release counter; the down rows of expert u
//      wait for that counter, so the down math of expert u overlaps the
//      gate/up stream of the experts after it;
//   4. combines sum_j w_j o_j for its down rows (fixed expert order), adds the
//      bf16 residual, and joins a grid-wide barrier before the next layer.
// All spin-waits are bounded by a deadline; on expiry the kernel records
// HFQ_ERR_TIMEOUT in the workspace status word and winds down.
#include <cfloat>

#include "device.cuh"
#include "gemv.cuh"
#include "ptx.cuh"
#include "sync.cuh"
#include "topk.cuh"

namespace hfq {
namespace {

constexpr int kCW = 8;                  // consumer warps
constexpr int kThr = (kCW + 1) * 32;    // + one producer warp
constexpr int kStage = 17408;           // ring stage bytes (16 rows of 1088 bytes)
constexpr int kMaxStages = 16;
constexpr int kMaxT = 8;
constexpr int kMaxU = 128;              // unique experts per layer (T*k <= 128)
constexpr int kMaxRowsW = 4;            // down rows owned by one consumer warp
constexpr int kMaxHChunks = 2;          // 16-element h chunks per lane (I <= 1024)
constexpr int kHsPairs = 16;            // (token, expert) h vectors staged per batch
constexpr int kStamps = 32;             // timeline stamps per layer
constexpr int kMaxCopies = 512;         // bulk copies per layer and CTA
constexpr int kSmemOptin = 232448;      // 227 KB per CTA on sm_100 (static + dynamic)
constexpr int kSmemLimit = kSmemOptin - 4096;   // dynamic budget, leaving room for static

struct StackArgs {
    const void *const *eptr[HFQ_MAX_STACK_LAYERS];
    const uint8_t *eloc[HFQ_MAX_STACK_LAYERS];
    const float *logits;      // [L][T][E], or null when the routing is given
    const int32_t *idx_in;    // [T][k] given routing (single layer) or null
    const float *wts_in;
    const void *x0;           // [T][H], bf16 (or f32 when x0_f32)
    uint16_t *x_out;          // [T][H] bf16 residual after the last layer, or null
    uint16_t *xbuf;           // [2][T][H] bf16 ping-pong
    float *h;                 // [T*k][Ip]
    float *y;                 // [L][T][H] or null
    uint16_t *y_bf16;         // [T][H] (last layer) or null
    int32_t *idx_all;         // [L][T][k] or null
    float *wts_all;
    unsigned *ctl;            // status, done counter, barriers, h counters
    long long timeout_ns;
    int L, T, E, k, H, I;
    int x0_f32;
    int n_stages;
    int extra_arrivals;       // test hook: grid barriers wait for this many more CTAs
    unsigned long long *timeline;   // debug: [2][L][kStamps] %globaltimer stamps, or null
};

struct Shared {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    int sel[kMaxT][HFQ_MAX_TOPK];
    float wsel[kMaxT][HFQ_MAX_TOPK];
    unsigned ebits[HFQ_MAX_EXPERTS / 32];
    int U;
    int abort;
    int last_cta;
    int uexp[kMaxU];
    unsigned umask[kMaxU];
    signed char ujt[kMaxU][kMaxT];
    float uw[kMaxU][kMaxT];
    int upair0[kMaxU + 1];                  // first pair slot of each expert (expert-major)
    int pair_row[kMaxU * kMaxT];            // h row (t*k + j) of each pair slot
    const uint8_t *ubase[kMaxU];            // base address of each selected expert
    unsigned char uloc[kMaxU];              // 1 = host-mapped
    int4 copies[kMaxCopies];                // {src offset, bytes, dst offset, stage << 8 | u}
    int ncopies;
    int Ul[HFQ_MAX_STACK_LAYERS];
};

struct Geo {
    int H, I, T, k, E, G, c;
    int nbH, nbI, Hp, Ip;
    int rowB_gu, rowB_d;
    size_t mg;                   // bytes of one gate (or up) matrix
    int n_gu, n_d;               // rows per item
    int HxRow, HsRow;            // padded smem rows of x (per token) and h (per pair)
    int gu_lo, gu_hi, d_lo, d_hi;
};

__device__ __forceinline__ Geo make_geo(const StackArgs &a)
{
    Geo g;
    g.H = a.H; g.I = a.I; g.T = a.T; g.k = a.k; g.E = a.E;
    g.G = gridDim.x; g.c = blockIdx.x;
    g.nbH = (a.H + kBlock - 1) / kBlock;
    g.nbI = (a.I + kBlock - 1) / kBlock;
    g.Hp = g.nbH * kBlock;
    g.Ip = g.nbI * kBlock;
    g.rowB_gu = g.nbH * kBlockBytes;
    g.rowB_d = g.nbI * kBlockBytes;
    g.mg = (size_t)a.I * g.rowB_gu;
    g.n_gu = (kStage / 2 - 16) / g.rowB_gu;
    g.n_d = (kStage - 16) / g.rowB_d;
    g.HxRow = g.Hp + 2 * (g.Hp >> 6);    // xpad(): +2 floats per 64 columns
    g.HsRow = g.Ip / 16 * 20;            // 16 values + 4 pad per chunk: conflict-free LDS.128
    g.gu_lo = (int)((long long)g.c * a.I / g.G);
    g.gu_hi = (int)((long long)(g.c + 1) * a.I / g.G);
    g.d_lo = (int)((long long)g.c * a.H / g.G);
    g.d_hi = (int)((long long)(g.c + 1) * a.H / g.G);
    return g;
}

// ------------------------------------------------------------ item sequence
// Units in consumption order: GU(0) .. GU(U-1), then D(0) .. D(U-1).  Units
// split into items of at most n_gu (n_d) rows; items pack into ring stages
// first-fit in order, so the down bytes are prefetched while the gate/up rows
// are computed.  Producer and consumers run the same generator, so no table
// is stored.
struct Item {
    int type;          // 0 = gate/up, 1 = down
    int u, q;          // unique-expert index, unit index
    int r0, n;         // first row, rows
    int stage;         // stage index within the layer
    int off0, off1;    // byte offsets of the two copies in the stage
    int len0, len1;    // copy lengths (multiples of 16)
    int dl0, dl1;      // data start within the copy (0 or 8)
    uint32_t src0, src1;   // 16-aligned source offsets within the expert
};

struct Gen {
    int q, sub, stage, fill, U;
};

__device__ __forceinline__ void unit_of(int q, int U, int &type, int &u)
{
    type = q >= U;
    u = type ? q - U : q;
}

__device__ __forceinline__ void span16(uint32_t off, uint32_t len, uint32_t &a16, int &len16,
                                       int &delta)
{
    a16 = off & ~15u;
    uint32_t e16 = (off + len + 15u) & ~15u;
    len16 = (int)(e16 - a16);
    delta = (int)(off - a16);
}

__device__ bool next_item(Gen &g, const Geo &geo, Item &it)
{
    while (g.q < 2 * g.U) {
        int type, u;
        unit_of(g.q, g.U, type, u);
        const int lo = type ? geo.d_lo : geo.gu_lo, hi = type ? geo.d_hi : geo.gu_hi;
        const int nmax = type ? geo.n_d : geo.n_gu;
        const int r0 = lo + g.sub * nmax;
        if (r0 >= hi) { ++g.q; g.sub = 0; continue; }
        const int n = min(nmax, hi - r0);
        ++g.sub;
        it.type = type; it.u = u; it.q = g.q; it.r0 = r0; it.n = n;
        int need;
        if (type == 0) {
            span16((uint32_t)r0 * geo.rowB_gu, (uint32_t)n * geo.rowB_gu, it.src0, it.len0, it.dl0);
            span16((uint32_t)(geo.mg + (size_t)r0 * geo.rowB_gu), (uint32_t)n * geo.rowB_gu, it.src1,
                   it.len1, it.dl1);
            need = it.len0 + it.len1;
        } else {
            span16((uint32_t)(2 * geo.mg + (size_t)r0 * geo.rowB_d), (uint32_t)n * geo.rowB_d,
                   it.src0, it.len0, it.dl0);
            it.len1 = 0; it.dl1 = 0; it.src1 = 0;
            need = it.len0;
        }
        if (g.fill + need > kStage) { ++g.stage; g.fill = 0; }
        it.stage = g.stage;
        it.off0 = g.fill;
        it.off1 = g.fill + it.len0;
        g.fill += need;
        return true;
    }
    return false;
}

// ---------------------------------------------------------------- waiting
__device__ __forceinline__ WaitCtx wctx(const StackArgs &a, Shared &sh)
{
    return WaitCtx{a.ctl, a.timeout_ns, &sh.abort};
}

__device__ __forceinline__ bool wait_counter(const StackArgs &a, Shared &sh, const unsigned *p, unsigned target)
{
    return wait_counter_ge(wctx(a, sh), p, target);
}

__device__ __forceinline__ bool wait_mbar(const StackArgs &a, Shared &sh, uint64_t *bar, uint32_t parity)
{
    return wait_mbar_phase(wctx(a, sh), bar, parity);
}

// ---------------------------------------------------------------- routing
// Top-k of one token by one warp; lanes j < k also fetch the base address of
// the j-th selected expert when `ubase` is given.
template <int M>
__device__ void warp_topk(const float *__restrict__ row, int E, int k, int *sel, float *wsel,
                          const void *const *eptr, const uint8_t *eloc, const uint8_t **ubase,
                          unsigned char *uloc)
{
    const int lane = threadIdx.x & 31;
    int my_e;
    float my_w;
    warp_topk_rounds<M>(row, E, k, my_e, my_w, [](int, int) {});
    if (lane < k) {
        if (ubase) {
            ubase[lane] = static_cast<const uint8_t *>(eptr[my_e]);
            uloc[lane] = eloc ? eloc[my_e] : 0;
        }
        sel[lane] = my_e;
        wsel[lane] = my_w;
    }
}

// ubase/uloc (nullable): for a single token, slot j's expert base address and
// location are fetched here, in slot order.
__device__ void route_token(const float *row, int E, int k, int *sel, float *wsel,
                            const void *const *eptr = nullptr, const uint8_t *eloc = nullptr,
                            const uint8_t **ubase = nullptr, unsigned char *uloc = nullptr)
{
    if (E <= 32) warp_topk<1>(row, E, k, sel, wsel, eptr, eloc, ubase, uloc);
    else if (E <= 64) warp_topk<2>(row, E, k, sel, wsel, eptr, eloc, ubase, uloc);
    else if (E <= 128) warp_topk<4>(row, E, k, sel, wsel, eptr, eloc, ubase, uloc);
    else if (E <= 256) warp_topk<8>(row, E, k, sel, wsel, eptr, eloc, ubase, uloc);
    else warp_topk<16>(row, E, k, sel, wsel, eptr, eloc, ubase, uloc);
}

// Unique experts of the layer, ascending; per (u, t) the slot j (or -1).
__device__ void build_table(Shared &sh, int T, int k)
{
    const int lane = threadIdx.x & 31;
    if (lane < HFQ_MAX_EXPERTS / 32) sh.ebits[lane] = 0u;
    for (int i = lane; i < kMaxU * kMaxT; i += 32) (&sh.ujt[0][0])[i] = -1;
    __syncwarp();
    for (int p = lane; p < T * k; p += 32) {
        int e = sh.sel[p / k][p % k];
        atomicOr(&sh.ebits[e >> 5], 1u << (e & 31));
    }
    __syncwarp();
    int cnt = lane < HFQ_MAX_EXPERTS / 32 ? __popc(sh.ebits[lane]) : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int base = incl - cnt;
    int total = __shfl_sync(0xffffffffu, incl, 31);
    __shared__ int wbase[HFQ_MAX_EXPERTS / 32];
    if (lane < HFQ_MAX_EXPERTS / 32) wbase[lane] = base;
    for (int u = lane; u < kMaxU; u += 32) sh.umask[u] = 0u;
    __syncwarp();
    for (int p = lane; p < T * k; p += 32) {
        int t = p / k, j = p % k;
        int e = sh.sel[t][j];
        int u = wbase[e >> 5] + __popc(sh.ebits[e >> 5] & ((1u << (e & 31)) - 1u));
        sh.uexp[u] = e;
        sh.ujt[u][t] = (signed char)j;
        sh.uw[u][t] = sh.wsel[t][j];
        atomicOr(&sh.umask[u], 1u << t);
    }
    if (lane == 0) sh.U = total;
    __syncwarp();
}

// One token: the k slots are the unique experts, in slot order.
__device__ void build_table_t1(Shared &sh, int k)
{
    const int lane = threadIdx.x & 31;
    if (lane < k) {
        sh.uexp[lane] = sh.sel[0][lane];
        sh.umask[lane] = 1u;
        sh.ujt[lane][0] = (signed char)lane;
        sh.uw[lane][0] = sh.wsel[0][lane];
    }
    if (lane == 0) sh.U = k;
    __syncwarp();
}

// Pair slots (expert-major, tokens ascending), their h rows, and every
// selected expert's base address and location, fetched in one round of loads.
__device__ void finish_table(Shared &sh, int k, const void *const *eptr, const uint8_t *eloc,
                             bool have_bases)
{
    const int lane = threadIdx.x & 31, U = sh.U;
    if (lane == 0) {
        int n = 0;
        for (int u = 0; u < U; ++u) {
            sh.upair0[u] = n;
            unsigned m = sh.umask[u];
            while (m) {
                const int t = __ffs(m) - 1;
                m &= m - 1;
                sh.pair_row[n++] = t * k + sh.ujt[u][t];
            }
        }
        sh.upair0[U] = n;
    }
    for (int u = lane; !have_bases && u < U; u += 32) {
        const int e = sh.uexp[u];
        sh.ubase[u] = static_cast<const uint8_t *>(eptr[e]);
        sh.uloc[u] = eloc ? eloc[e] : 0;
    }
    __syncwarp();
}

// ----------------------------------------------------------------- kernel
__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory"); }

__device__ __forceinline__ void stamp(const StackArgs &a, int which, int l, int s)
{
    if (a.timeline && threadIdx.x == 0 && l < a.L) {
        const int G = gridDim.x;
        const int slot = blockIdx.x == 0 ? 0 : (blockIdx.x == G / 2 ? 1 : -1);
        if (slot >= 0) a.timeline[((size_t)slot * a.L + l) * kStamps + s] = globaltimer_ns();
    }
    (void)which;
}

template <int MAXT>
__global__ void __launch_bounds__(kThr, 1) stack_kernel(const __grid_constant__ StackArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const Geo geo = make_geo(a);
    const int NS = a.n_stages;
    uint8_t *ring = smem;
    float *xs = reinterpret_cast<float *>(smem + (size_t)NS * kStage);          // [T][HxRow]
    float *hs = xs + ((size_t)a.T * geo.HxRow + 3) / 4 * 4;                    // [kHsPairs][HsRow]
    Shared &sh = *reinterpret_cast<Shared *>(reinterpret_cast<uint8_t *>(hs) +
                                             (size_t)kHsPairs * geo.HsRow * 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], kCW);
        }
        sh.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    int stage_base = 0;          // ring stages used by earlier layers (same in every warp)
    float2 xr[MAXT == 1 ? 32 : 1];   // this lane's 64 activations (T = 1)
    for (int l = 0; l < a.L; ++l) {
        stamp(a, 0, l, 0);
        // ---------------------------------------------- 1. route + load x
        // Routing runs on the last T consumer warps; the others start loading the
        // layer input meanwhile.  Layer l's logits are read only here, after the
        // grid barrier that ends layer l-1.
        const void *xin = l == 0 ? a.x0 : (const void *)(a.xbuf + (size_t)(l & 1) * a.T * a.H);
        const bool xin_f32 = l == 0 && a.x0_f32;
        const int route_w0 = kCW - a.T;
        if (warp >= route_w0 && warp < kCW && !sh.abort) {
            const int t = warp - route_w0;
            if (a.idx_in) {
                for (int j = lane; j < a.k; j += 32) {
                    int e = a.idx_in[t * a.k + j];
                    if ((unsigned)e >= (unsigned)a.E) {
                        // a caller's id outside [0, E): recorded; expert 0 stands
                        // in so that every table index stays in range
                        atomicCAS(a.ctl, 0u, (unsigned)HFQ_ERR_ARG);
                        e = 0;
                    }
                    sh.sel[t][j] = e;
                    sh.wsel[t][j] = a.wts_in[t * a.k + j];
                }
            } else {
                if constexpr (MAXT == 1)
                    route_token(a.logits + ((size_t)l * a.T + t) * a.E, a.E, a.k, sh.sel[t],
                                sh.wsel[t], a.eptr[l], a.eloc[l], sh.ubase, sh.uloc);
                else
                    route_token(a.logits + ((size_t)l * a.T + t) * a.E, a.E, a.k, sh.sel[t],
                                sh.wsel[t]);
            }
        }
        if (warp < kCW) {
            // layer input -> xs (f32, padded rows), once per CTA: every thread
            // issues all its 16-byte loads (8 bf16 or 4 f32 each) before using any
            constexpr int kMaxLoads = MAXT;              // T * Hp * 2 bytes / 4 KB <= T
            const int per = xin_f32 ? 4 : 8;             // values per 16-byte load
            const int nld = a.T * geo.Hp / per;          // loads for the whole [T][Hp] tile
            uint4 v[kMaxLoads * 2];
#pragma unroll
            for (int q = 0; q < kMaxLoads * 2; ++q) {
                const int i = tid + q * kCW * 32;
                v[q] = make_uint4(0u, 0u, 0u, 0u);
                if (i < nld) {
                    const int t = (i * per) / geo.Hp, c = i * per - t * geo.Hp;
                    if (c < a.H) {
                        const size_t o = (size_t)t * a.H + c;
                        v[q] = xin_f32 ? __ldcg(reinterpret_cast<const uint4 *>(static_cast<const float *>(xin) + o))
                                       : __ldcg(reinterpret_cast<const uint4 *>(static_cast<const unsigned short *>(xin) + o));
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < kMaxLoads * 2; ++q) {
                const int i = tid + q * kCW * 32;
                if (i < nld) {
                    const int t = (i * per) / geo.Hp, c = i * per - t * geo.Hp;
                    float2 *dst = reinterpret_cast<float2 *>(xs + (size_t)t * geo.HxRow + xpad(c));
                    if (xin_f32) {
                        dst[0] = make_float2(__uint_as_float(v[q].x), __uint_as_float(v[q].y));
                        dst[1] = make_float2(__uint_as_float(v[q].z), __uint_as_float(v[q].w));
                    } else {
                        const uint32_t w4[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
                        for (int r = 0; r < 4; ++r)
                            dst[r] = make_float2(__uint_as_float(w4[r] << 16),
                                                 __uint_as_float(w4[r] & 0xFFFF0000u));
                    }
                }
            }
        }
        __syncthreads();
        stamp(a, 1, l, 1);
        if (warp == 0) {
            if (MAXT == 1) build_table_t1(sh, a.k);
            else build_table(sh, a.T, a.k);
            // one token routed here: the routing warp already fetched the bases
            finish_table(sh, a.k, a.eptr[l], a.eloc[l], MAXT == 1 && !a.idx_in);
        }
        __syncthreads();
        stamp(a, 2, l, 2);
        const int U = sh.U;
        if (tid == 0 && l < HFQ_MAX_STACK_LAYERS) sh.Ul[l] = U;
        if (a.idx_all && blockIdx.x == 0 && warp < a.T && lane < a.k) {
            a.idx_all[((size_t)l * a.T + warp) * a.k + lane] = sh.sel[warp][lane];
            a.wts_all[((size_t)l * a.T + warp) * a.k + lane] = sh.wsel[warp][lane];
        }
        unsigned *hdone = a.ctl + kCtlH + (size_t)l * kCtlHStride;     // CTAs whose h rows are written
        int n_stages_layer = 0;

        if (warp == kCW) {
            // ------------------------------------------ 2. producer warp
            // First the layer's whole copy list (no issue yet: the consumers are
            // idle and the generator runs undisturbed), then one tight issue loop.
            Gen g{0, 0, 0, 0, U};
            Item it;
            int nc = 0;
            bool more;
            while ((more = next_item(g, geo, it)) && nc + 2 <= kMaxCopies) {
                if (lane == 0) {
                    sh.copies[nc] = make_int4((int)it.src0, it.len0, it.off0, (it.stage << 8) | it.u);
                    if (it.type == 0)
                        sh.copies[nc + 1] = make_int4((int)it.src1, it.len1, it.off1, (it.stage << 8) | it.u);
                }
                nc += it.type == 0 ? 2 : 1;
            }
            if (more && lane == 0) {              // excluded on the host (stack_supported)
                sh.abort = 1;
                atomicCAS(a.ctl, 0u, (unsigned)HFQ_ERR_UNSUPPORTED);
            }
            __syncwarp();
            int cur = -1, slot = 0;
            for (int ci = 0; ci < nc && !sh.abort; ++ci) {
                const int4 c = sh.copies[ci];
                const int stage = c.w >> 8, u = c.w & 0xFF;
                if (stage != cur) {
                    if (cur >= 0 && lane == 0) mbar_arrive(&sh.full[slot]);
                    cur = stage;
                    const int seq = stage_base + cur;
                    slot = seq % NS;
                    if (seq >= NS && !wait_mbar(a, sh, &sh.empty[slot], ((seq / NS) - 1) & 1)) break;
                    fence_proxy_async_smem();
                }
                const uint8_t *src = sh.ubase[u] + (uint32_t)c.x;
                if (((uintptr_t)src & 15u) != 0) {          // bulk copies start on 16 bytes
                    if (lane == 0) { atomicCAS(a.ctl, 0u, (unsigned)HFQ_ERR_ARG); sh.abort = 1; }
                    break;
                }
                uint8_t *dst = ring + (size_t)slot * kStage + c.z;
                const int len = c.y;
                if (!sh.uloc[u]) {
                    if (lane == 0) {
                        mbar_expect_tx(&sh.full[slot], (uint32_t)len);
                        bulk_g2s(dst, src, (uint32_t)len, &sh.full[slot]);
                    }
                } else {
                    // host-mapped expert: 16-byte loads over PCIe, four in flight per lane
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
            }
            if (cur >= 0 && lane == 0) mbar_arrive(&sh.full[slot]);
            n_stages_layer = g.stage + (g.fill > 0 ? 1 : 0);
            if (a.timeline && lane == 0 && n_stages_layer <= NS) {
                // debug timeline: when this CTA's stages land (the producer is idle now)
                const int who = blockIdx.x == 0 ? 0 : (blockIdx.x == (int)gridDim.x / 2 ? 1 : -1);
                if (who >= 0) {
                    unsigned long long *tl = a.timeline + ((size_t)who * a.L + l) * kStamps;
                    tl[21] = globaltimer_ns();
                    for (int st = 0; st < n_stages_layer && st < 10; ++st) {
                        const int seq = stage_base + st;
                        uint64_t t0 = globaltimer_ns();
                        while (!mbar_try_wait(&sh.full[seq % NS], (seq / NS) & 1) &&
                               !deadline_passed(t0, a.timeout_ns)) {
                        }
                        tl[22 + st] = globaltimer_ns();
                    }
                }
            }
        } else {
            // ------------------------------------------ 3. consumer warps
            float2 sx[MAXT];                        // (sum over even, sum over odd) per token
            const int pb = lane >> 2, pq = lane & 3;        // piece: block, quarter
            const bool has_piece = pb < geo.nbH;
            const int col0 = pb * kBlock + pq * 64;
            const int xcol0 = xpad(col0);                   // padded smem column
#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                sx[t] = make_float2(0.f, 0.f);
                if (t < a.T && has_piece) {
                    const float2 *xp = reinterpret_cast<const float2 *>(xs + (size_t)t * geo.HxRow + xcol0);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float2 v = xp[i];
                        if constexpr (MAXT == 1) xr[i] = v;
                        sx[t].x += v.x;
                        sx[t].y += v.y;
                    }
                }
            }
            float acc[kMaxRowsW][MAXT];
#pragma unroll
            for (int r = 0; r < kMaxRowsW; ++r)
#pragma unroll
                for (int t = 0; t < MAXT; ++t) acc[r][t] = 0.0f;

            Gen g{0, 0, 0, 0, U};
            Item it;
            int cur = -1, slot = 0, gu_rows_seen = 0;
            bool dead = sh.abort != 0, announced = false, first_stage = true;
            int batch_u0 = 0, batch_u1 = 0;          // experts whose h is staged in hs
            const int nch = geo.nbI * 16;            // 8-byte chunks per down row
            // h of this CTA's gate/up rows is complete: one release per CTA
            auto announce = [&]() {
                consumer_bar();
                stamp(a, 4, l, 16);
                if (tid == 0) { __threadfence(); red_release_gpu_add(hdone, 1u); }
                announced = true;
            };
            while (next_item(g, geo, it)) {
                dead = dead || sh.abort != 0;
                if (it.type == 1 && !announced) {
                    announce();
                    // wait until every CTA has written its h rows
                    int ok = 1;
                    if (tid == 0 && !dead) ok = wait_counter(a, sh, hdone, (unsigned)geo.G) ? 1 : 0;
                    if (tid == 0 && !ok) sh.abort = 1;
                    stamp(a, 5, l, 17);
                    consumer_bar();
                    dead = dead || sh.abort != 0;
                }
                if (it.stage != cur) {
                    if (cur >= 0 && lane == 0) mbar_arrive(&sh.empty[slot]);
                    cur = it.stage;
                    slot = (stage_base + cur) % NS;
                    if (!dead && !wait_mbar(a, sh, &sh.full[slot], ((stage_base + cur) / NS) & 1))
                        dead = true;
                    if (cur < 12) stamp(a, 3, l, 3 + cur);
                    (void)first_stage;
                }
                const uint8_t *sbase = ring + (size_t)slot * kStage;
                const int u = it.u;
                const unsigned um = sh.umask[u];
                if (it.type == 0) {
                    // gate/up rows, round-robin over the consumer warps
                    for (int i = 0; i < it.n; ++i, ++gu_rows_seen) {
                        if (dead || gu_rows_seen % kCW != warp) continue;
                        const uint8_t *grow = sbase + it.off0 + it.dl0 + (size_t)i * geo.rowB_gu;
                        const uint8_t *urow = sbase + it.off1 + it.dl1 + (size_t)i * geo.rowB_gu;
                        float gd[MAXT], ud[MAXT];
#pragma unroll
                        for (int t = 0; t < MAXT; ++t) { gd[t] = 0.f; ud[t] = 0.f; }
                        if (has_piece) {
                            const uint8_t *gb = grow + pb * kBlockBytes, *ub = urow + pb * kBlockBytes;
                            const float2 gsz = *reinterpret_cast<const float2 *>(gb);
                            const float2 usz = *reinterpret_cast<const float2 *>(ub);
                            uint32_t gw[8], uw[8];
                            lds_words(gb + 8 + pq * 32, gw);
                            lds_words(ub + 8 + pq * 32, uw);
#pragma unroll
                            for (int t = 0; t < MAXT; ++t) {
                                if (!(um >> t & 1u)) continue;
                                const float2 *xp = MAXT == 1 ? xr
                                    : reinterpret_cast<const float2 *>(xs + (size_t)t * geo.HxRow + xcol0);
                                gd[t] = finish_dot(nib64_fma(gw, xp), sx[t], gsz.x, gsz.y);
                                ud[t] = finish_dot(nib64_fma(uw, xp), sx[t], usz.x, usz.y);
                            }
                        }
                        const int r = it.r0 + i;
#pragma unroll
                        for (int t = 0; t < MAXT; ++t) {
                            if (!(um >> t & 1u)) continue;
                            float gv = warp_sum(gd[t]), uv = warp_sum(ud[t]);
                            if (lane == 0) {
                                const int p = t * a.k + sh.ujt[u][t];
                                a.h[(size_t)p * geo.Ip + r] = silu(gv) * uv;
                            }
                        }
                    }
                } else {
                    // down rows of expert u; stage the h vectors of a batch of experts
                    // (at most kHsPairs (token, expert) pairs) with one round of loads
                    if (u >= batch_u1) {
                        batch_u0 = u;
                        batch_u1 = u + 1;
                        while (batch_u1 < U && sh.upair0[batch_u1 + 1] - sh.upair0[batch_u0] <= kHsPairs)
                            ++batch_u1;
                        consumer_bar();                    // previous batch no longer read
                        const int p0 = sh.upair0[batch_u0];
                        const int nv4 = (sh.upair0[batch_u1] - p0) * (geo.Ip / 4);
                        const int per_pair = geo.Ip / 4;
                        for (int i0 = tid; !dead && i0 < nv4; i0 += 4 * kCW * 32) {
                            float4 v[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int i = i0 + q * kCW * 32;
                                v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                                if (i < nv4) {
                                    const int ps = i / per_pair, c = (i - ps * per_pair) * 4;
                                    if (c < a.I)
                                        v[q] = __ldcg(reinterpret_cast<const float4 *>(
                                            a.h + (size_t)sh.pair_row[p0 + ps] * geo.Ip + c));
                                }
                            }
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int i = i0 + q * kCW * 32;
                                if (i < nv4) {
                                    const int ps = i / per_pair, c = (i - ps * per_pair) * 4;
                                    *reinterpret_cast<float4 *>(hs + (size_t)ps * geo.HsRow +
                                                                (c >> 4) * 20 + (c & 15)) = v[q];
                                }
                            }
                        }
                        consumer_bar();
                        stamp(a, 0, l, 18);
                    }
                    const int slot0 = sh.upair0[u] - sh.upair0[batch_u0];   // first pair slot of u
                    if (!dead) {
                        // T = 1: this lane's h chunks and their sums, loaded once for the
                        // item; T > 1: read per row from shared memory (registers)
                        constexpr int kHT = MAXT == 1 ? 1 : 1;
                        float2 hv[kHT][kMaxHChunks][8];
                        float2 hsum[kHT][kMaxHChunks];
                        if constexpr (MAXT == 1) {
#pragma unroll
                            for (int m = 0; m < kMaxHChunks; ++m) {
                                const int c = lane + 32 * m;
                                hsum[0][m] = make_float2(0.f, 0.f);
                                const bool ok = c < nch && c * 16 < a.I;
                                const float2 *hp = reinterpret_cast<const float2 *>(
                                    hs + (size_t)slot0 * geo.HsRow + (ok ? c : 0) * 20);
#pragma unroll
                                for (int v = 0; v < 8; ++v) {
                                    hv[0][m][v] = ok ? hp[v] : make_float2(0.f, 0.f);
                                    hsum[0][m].x += hv[0][m][v].x;
                                    hsum[0][m].y += hv[0][m][v].y;
                                }
                            }
                        }
                        // the rows of this item that this warp owns, as independent chains
#pragma unroll
                        for (int rs = 0; rs < kMaxRowsW; ++rs) {
                            const int r = geo.d_lo + warp + rs * kCW;
                            if (r < it.r0 || r >= it.r0 + it.n) continue;
                            const uint8_t *row = sbase + it.off0 + it.dl0 + (size_t)(r - it.r0) * geo.rowB_d;
#pragma unroll
                            for (int m = 0; m < kMaxHChunks; ++m) {
                                const int c = lane + 32 * m;
                                if (c >= nch || c * 16 >= a.I) continue;
                                const uint8_t *blk = row + (c >> 4) * kBlockBytes;
                                const float2 sz = *reinterpret_cast<const float2 *>(blk);
                                const uint2 nv = *reinterpret_cast<const uint2 *>(blk + 8 + (c & 15) * 8);
                                if constexpr (MAXT == 1) {
                                    const float part = finish_dot(nib16_fma(nv, hv[0][m]), hsum[0][m], sz.x, sz.y);
                                    acc[rs][0] = fmaf(sh.uw[u][0], part, acc[rs][0]);
                                } else {
                                    int ps = slot0;
#pragma unroll
                                    for (int t = 0; t < MAXT; ++t) {
                                        if (!((um >> t) & 1u)) continue;
                                        const float2 *hp = reinterpret_cast<const float2 *>(
                                            hs + (size_t)ps * geo.HsRow + c * 20);
                                        ++ps;
                                        float2 h8[8];
                                        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
                                        for (int v = 0; v < 8; ++v) {
                                            h8[v] = hp[v];
                                            s2.x += h8[v].x;
                                            s2.y += h8[v].y;
                                        }
                                        const float part = finish_dot(nib16_fma(nv, h8), s2, sz.x, sz.y);
                                        acc[rs][t] = fmaf(sh.uw[u][t], part, acc[rs][t]);
                                    }
                                }
                            }
                        }
                    }
                }
            }
            if (cur >= 0 && lane == 0) mbar_arrive(&sh.empty[slot]);
            if (!announced) announce();            // a CTA without down rows still announces
            stamp(a, 6, l, 19);
            if (dead) sh.abort = 1;
            // ------------------------------------------ 4. combine + residual
            if (!dead) {
                uint16_t *xo = l == a.L - 1 ? a.x_out
                                            : a.xbuf + (size_t)((l + 1) & 1) * a.T * a.H;
#pragma unroll
                for (int rs = 0; rs < kMaxRowsW; ++rs) {
                    const int r = geo.d_lo + warp + rs * kCW;
                    if (r >= geo.d_hi) break;
#pragma unroll
                    for (int t = 0; t < MAXT; ++t) {
                        if (t >= a.T) break;
                        const float y = warp_sum(acc[rs][t]);
                        if (lane == 0) {
                            const size_t o = (size_t)t * a.H + r;
                            if (a.y) a.y[(size_t)l * a.T * a.H + o] = y;
                            if (a.y_bf16 && l == a.L - 1) a.y_bf16[o] = float_to_bf16_bits(y);
                            const float xv = xs[(size_t)t * geo.HxRow + xpad(r)];
                            if (xo) xo[o] = float_to_bf16_bits(xv + y);
                        }
                    }
                }
            }
        }
        // every warp computed the same stage count; the producer's is authoritative
        __shared__ int s_nst;
        if (warp == kCW && lane == 0) s_nst = n_stages_layer;
        __syncthreads();
        stamp(a, 7, l, 20);
        stage_base += s_nst;
        // ---------------------------------------------- 5. grid barrier
        if (l + 1 < a.L) {
            if (tid == 0) {
                unsigned *bar = a.ctl + kCtlBar + l;
                __threadfence();
                red_release_gpu_add(bar, 1u);
                if (!sh.abort && !wait_counter(a, sh, bar, (unsigned)(geo.G + a.extra_arrivals)))
                    sh.abort = 1;
            }
            __syncthreads();
        }
    }
    // make sure no bulk copy into this CTA's shared memory is still in flight
    if (warp == kCW && lane == 0) {
        for (int s = 0; s < NS; ++s) {
            const int seq = stage_base - 1 - s;
            if (seq < 0) break;
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&sh.full[seq % NS], (seq / NS) & 1) &&
                   !deadline_passed(t0, a.timeout_ns)) {
            }
        }
    }
    // the last CTA to finish clears the counters this launch used
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        unsigned old = atomicAdd(a.ctl + kCtlDone, 1u);
        sh.last_cta = old == (unsigned)geo.G - 1;
    }
    __syncthreads();
    if (sh.last_cta) {
        __threadfence();
        if (*(volatile unsigned *)a.ctl == 0u) {
            for (int l = tid; l < a.L && l < HFQ_MAX_STACK_LAYERS; l += kThr) {
                a.ctl[kCtlBar + l] = 0u;
                a.ctl[kCtlH + (size_t)l * kCtlHStride] = 0u;
            }
            __syncthreads();
            if (tid == 0) { __threadfence(); a.ctl[kCtlDone] = 0u; }
        }
    }
}

size_t smem_for(int T, int H, int I, int n_stages, int maxt)
{
    size_t Hp = (size_t)(H + kBlock - 1) / kBlock * kBlock, Ip = (size_t)(I + kBlock - 1) / kBlock * kBlock;
    const size_t HxRow = Hp + 2 * (Hp >> 6), HsRow = Ip / 16 * 20;
    const size_t xs = (size_t)T * HxRow * 4;
    (void)maxt;
    return (size_t)n_stages * kStage + (xs + 15) / 16 * 16 + (size_t)kHsPairs * HsRow * 4 +
           sizeof(Shared);
}

}  // namespace

// SMs of the current device; 0 when there is none (callers then fail with
// HFQ_ERR_CUDA instead of sizing a grid from it).
int sm_count()
{
    static int n = 0;
    if (n <= 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            n = v;
        else
            cudaGetLastError();                 // the failed query's error is not left for a later check
    }
    return n > 0 ? n : 0;
}

// Whether the persistent kernel handles this shape (else the per-layer path).
bool stack_supported(int T, int H, int I, int k, int G)
{
    if (T < 1 || T > kMaxT || T * k > kMaxU) return false;
    if (expert_bytes(H, I) % 16) return false;                  // 16-byte aligned experts
    if (H > 2048 || I > 1024) return false;                     // lane slices in registers
    if ((H + G - 1) / G > kMaxRowsW * kCW) return false;
    // bulk copies of one layer in one CTA: two per gate/up item, one per down item
    {
        const int nbH = (H + kBlock - 1) / kBlock, nbI = (I + kBlock - 1) / kBlock;
        const int n_gu = (kStage / 2 - 16) / (nbH * kBlockBytes), n_d = (kStage - 16) / (nbI * kBlockBytes);
        if (n_gu < 1 || n_d < 1) return false;
        const int gu_rows = (I + G - 1) / G, d_rows = (H + G - 1) / G;
        const int per_u = 2 * ((gu_rows + n_gu - 1) / n_gu) + (d_rows + n_d - 1) / n_d;
        if (T * k * per_u > kMaxCopies) return false;
    }
    int maxt = T == 1 ? 1 : 8;
    return smem_for(T, H, I, 4, maxt) <= (size_t)kSmemLimit;
}

size_t stack_ctl_bytes() { return kCtlBytes; }

size_t stack_ctl_clear_bytes() { return kCtlWords * 4; }

hfq_status launch_stack(const hfq4_layer *layers, int L, const float *logits, const int32_t *idx_in,
                        const float *wts_in, const void *x0, bool x0_f32, int T, int k,
                        uint16_t *x_out, uint16_t *xbuf, float *h, float *y, uint16_t *y_bf16,
                        int32_t *idx_all, float *wts_all, unsigned *ctl, long long timeout_ns,
                        int extra_arrivals, cudaStream_t s)
{
    if (T == 1) {
        const hfq_status st = decode1_launch(layers, L, logits, idx_in, wts_in, x0, x0_f32, k, x_out, xbuf,
                                             h, y, y_bf16, idx_all, wts_all, ctl, timeout_ns,
                                             extra_arrivals, s);
        if (st != HFQ_ERR_UNSUPPORTED) return st;
    } else {
        const hfq_status st = verify_launch(layers, L, logits, idx_in, wts_in, x0, x0_f32, T, k, x_out, xbuf,
                                            h, y, y_bf16, idx_all, wts_all, ctl, timeout_ns, extra_arrivals, s);
        if (st != HFQ_ERR_UNSUPPORTED) return st;
    }
    StackArgs a;
    memset(&a, 0, sizeof a);
    for (int l = 0; l < L; ++l) {
        a.eptr[l] = layers[l].expert_ptr;
        a.eloc[l] = layers[l].expert_loc;
    }
    a.logits = logits; a.idx_in = idx_in; a.wts_in = wts_in; a.x0 = x0; a.x_out = x_out;
    a.xbuf = xbuf; a.h = h; a.y = y; a.y_bf16 = y_bf16; a.idx_all = idx_all; a.wts_all = wts_all;
    a.ctl = ctl; a.timeout_ns = timeout_ns; a.extra_arrivals = extra_arrivals;
    a.timeline = static_cast<unsigned long long *>(option_timeline());
    a.L = L; a.T = T; a.E = layers[0].n_experts; a.k = k; a.H = layers[0].hidden;
    a.I = layers[0].inter; a.x0_f32 = x0_f32 ? 1 : 0;
    const int maxt = T == 1 ? 1 : 8;
    int ns = kMaxStages;
    const void *fn = maxt == 1 ? (const void *)stack_kernel<1> : (const void *)stack_kernel<8>;
    static int dyn_limit[2] = {0, 0};
    if (!dyn_limit[maxt > 1]) {
        // the opt-in limit covers static + dynamic shared memory
        int dev = 0, optin = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, fn);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "stack kernel attributes: %s", cudaGetErrorString(e));
        int lim = optin - (int)fa.sharedSizeBytes;
        if (lim > kSmemLimit) lim = kSmemLimit;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "stack kernel attribute %d: %s", lim, cudaGetErrorString(e));
        dyn_limit[maxt > 1] = lim;
    }
    while (ns > 2 && smem_for(T, a.H, a.I, ns, maxt) > (size_t)dyn_limit[maxt > 1]) --ns;
    a.n_stages = ns;
    const size_t smem2 = smem_for(T, a.H, a.I, ns, maxt);
    if (smem2 > (size_t)dyn_limit[maxt > 1])
        return fail(HFQ_ERR_UNSUPPORTED, "stack kernel needs %zu bytes of shared memory", smem2);
    int resident = 0;
    cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, fn, kThr, smem2);
    if (oe != cudaSuccess || resident < 1)
        return fail(HFQ_ERR_UNSUPPORTED, "stack kernel: no CTA fits on an SM (%s, %zu bytes of "
                    "shared memory); the persistent launch needs one per SM",
                    cudaGetErrorString(oe), smem2);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sm_count());
    cfg.blockDim = dim3(kThr);
    cfg.dynamicSmemBytes = smem2;
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeCooperative;
    attrs[0].val.cooperative = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    void *params[] = {&a};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, params);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "stack kernel launch: %s", cudaGetErrorString(e));
    return HFQ_OK;
}

}  // namespace hfq
