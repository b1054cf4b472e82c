// verify.cu - persistent decode kernel for 2..8 tokens per step (speculative
// verify batches): every MoE layer of a step in one cooperative launch, one
// CTA of eight consumer warps and four producer warps per SM.
//
// hipfire thread, "HFQ quantisation format and GEMV": decode is a GEMV over
// 136-byte blocks, bound by the bytes of the selected experts; with T tokens a
// layer streams each unique selected expert once, whatever its token count.
// A CTA's share of expert u is fixed: rows [c*I/G, (c+1)*I/G) of its gate and
// up matrices and rows [c*H/G, (c+1)*H/G) of its down matrix.  Per layer:
//   1. warp t routes token t (softmax top-k, renormalised; hipfire offload
//      explainer, opening section) once layer l-1 has finished everywhere;
//      warp 0 lists the unique experts (ascending) and their (expert, token)
//      pairs, reading the layer's expert table from shared memory (copied in
//      while the previous layer's down items ran); all threads turn the T
//      inputs into per-64-value pieces of scaled bf16 pairs (gemv.cuh);
//   2. the producer warps stream one item per ring stage with 1-D bulk copies
//      (TMA, no multicast): the gate/up share of every unique expert, then its
//      down share; host-mapped experts are read with 16-byte loads (hipfire
//      offload explainer, "PCIe pass-through").  Items go round-robin to four
//      producer warps: one warp's consecutive bulk copies issue slowly while
//      many are in flight, several warps' copies overlap;
//   3. consumer warp w takes the pairs p = w, w + 8, ... : for a gate/up item
//      it computes all of the CTA's rows of its token at once (8 dots in
//      flight, one batched warp reduction) and writes h = silu(g) * u;
//   4. one release counter per layer makes every CTA's h visible (the down
//      bytes keep streaming meanwhile);
//   5. for a down item, the warp stages its pair's h (the next pair's loads in
//      flight meanwhile), computes the CTA's down rows and adds w_p * o into
//      its per-token row sums; the warps' sums are added in a fixed order,
//      the bf16 residual applied, and the CTA joins a grid barrier.
// Every wait is bounded (sync.cuh); on expiry the status word holds
// HFQ_ERR_TIMEOUT and every CTA winds down.
#include <algorithm>

#include "device.cuh"
#include "gemv.cuh"
#include "ptx.cuh"
#include "sync.cuh"
#include "topk.cuh"

namespace hfq {
namespace {

constexpr int kCW = 8;                  // consumer warps
constexpr int kPW = 4;                  // producer warps: stage s is filled by producer s % kPW
constexpr int kThr = (kCW + kPW) * 32;
constexpr int kMaxT = 8;
constexpr int kMaxP = 64;               // (expert, token) pairs per layer: T * k <= 64
constexpr int kMaxU = 64;
constexpr int kMaxNS = 24;              // ring stages
constexpr int kMaxDRows = 16;           // down rows per CTA
constexpr int kGuRows = 4;              // gate/up rows per batched warp reduction
constexpr int kPiece = 36;              // words per x piece: 32 bf16 pairs, exponent, f32 sum, 2 pad
constexpr int kHStride = 68;            // floats per staged 64-value h piece (bank spread)
constexpr int kSmemOptin = 232448;      // 227 KB per CTA on sm_100

struct VArgs {
    const void *const *eptr[HFQ_MAX_STACK_LAYERS];
    const uint8_t *eloc[HFQ_MAX_STACK_LAYERS];
    const float *logits;      // [L][T][E], or null when the routing is given
    const int32_t *idx_in;    // [T][k] given routing (single layer), or null
    const float *wts_in;
    const uint16_t *x0;       // [T][H] bf16
    uint16_t *x_out;          // [T][H] bf16 input of the layer after the last, or null
    uint16_t *xbuf;           // [2][T][H] bf16 ping-pong between layers (L > 1)
    float *h;                 // [T*k][Ip]: h of pair (t, j) at row t*k + j
    float *y;                 // [L][T][H], or null
    uint16_t *y_bf16;         // [T][H] of the last layer, or null
    int32_t *idx_all;         // [L][T][k], or null
    float *wts_all;
    unsigned *ctl;            // control block (device.cuh)
    long long timeout_ns;
    int L, T, E, k, H, I;
    int extra_arrivals;       // test hook: grid barriers wait for this many more CTAs
    int NS, stage_bytes;      // ring
    int xp_off, xres_off, ysh_off, hst_off, tab_off, sh_off;
    int tab_pref;             // the layers' expert tables are prefetched into shared memory
    unsigned long long *timeline;   // debug: [G][L][32] %globaltimer stamps, or null
};

struct VShared {
    uint64_t full[kMaxNS];
    uint64_t empty[kMaxNS];
    int sel[kMaxT][HFQ_MAX_TOPK];
    float wsel[kMaxT][HFQ_MAX_TOPK];
    unsigned ebits[HFQ_MAX_EXPERTS / 32];
    int wbase[HFQ_MAX_EXPERTS / 32];
    int U, P;
    int uexp[kMaxU];
    unsigned umask[kMaxU];
    signed char ujt[kMaxU][kMaxT];
    int pair0[kMaxU + 1];       // first pair of each unique expert
    int pt[kMaxP];              // token of pair p
    int prow[kMaxP];            // h row t*k + j of pair p
    float pw[kMaxP];            // routing weight of pair p
    const uint8_t *ubase[kMaxU];
    unsigned char uloc[kMaxU];
    int armed_seq[kMaxNS];      // latest item sequence number armed in each stage, or -1
    int abort;
    int last_cta;
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

// Debug timeline: stamp s of layer l for this CTA (ns of %globaltimer).
template <bool kOn>
__device__ __forceinline__ void vstamp(const VArgs &a, int l, int s, bool who)
{
    if (kOn && a.timeline && who && l < a.L)
        a.timeline[((size_t)blockIdx.x * a.L + l) * 32 + s] = globaltimer_ns();
}

// Debug: where a bounded wait of this kernel gave up, recorded once per
// launch into control words 3..5 (site, layer, item sequence) when the status
// word shows a timeout.
__device__ __forceinline__ void note_wait(const VArgs &a, bool ok, int site, int l, int seq)
{
    if (!ok && atomicCAS(a.ctl + 3, 0u, (unsigned)site) == 0u) {
        a.ctl[4] = (unsigned)l;
        a.ctl[5] = (unsigned)seq;
    }
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory"); }

// Lanes 8m..8m+7 hold values 8i..8i+7 (i = lane & 7) of one 64-value piece:
// the piece's largest magnitude and f32 sum (the butterfly adds the same pairs
// in every lane), then its scaled bf16 operand pairs into `piece` (kPiece
// words: 32 pair words, the scale exponent, the f32 sum).
__device__ __forceinline__ void build_x_piece(const float (&v)[8], uint32_t *piece)
{
    float m = 0.0f, s = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        m = fmaxf(m, fabsf(v[i]));
        s += v[i];
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        s += __shfl_xor_sync(0xffffffffu, s, o);
    }
    const int e = bf16_piece_scale(m);
    uint32_t X[4];
    bf16_x_pairs(v, e, X);
    const int i = threadIdx.x & 7;
    *reinterpret_cast<uint4 *>(piece + 4 * i) = make_uint4(X[0], X[1], X[2], X[3]);
    if (i == 0) {
        piece[32] = (uint32_t)e;
        piece[33] = __float_as_uint(s);
    }
}

// Warp 0: unique experts of the layer (ascending), their token masks and slot
// per token, and the pairs in (expert, token) order.
// Layer l's expert table (and location table) into shared memory, one
// cp.async group of warp 0, waited for in build_pairs: the table of the next
// layer travels while this one's down items compute.
__device__ __forceinline__ void fetch_tables(const VArgs &a, int l, uint8_t *tab)
{
    const int lane = threadIdx.x & 31;
    const uint8_t *src = reinterpret_cast<const uint8_t *>(a.eptr[l]);
    for (int i = lane; i < a.E / 2; i += 32) cp_async16(tab + 16 * i, src + 16 * i);
    if (a.eloc[l])
        for (int i = lane; i < a.E / 16; i += 32) cp_async16(tab + (size_t)a.E * 8 + 16 * i, a.eloc[l] + 16 * i);
    cp_async_commit();
}

__device__ void build_pairs(VShared &sh, const VArgs &a, int l, const uint8_t *tab)
{
    const int lane = threadIdx.x & 31, T = a.T, k = a.k;
    if (lane < HFQ_MAX_EXPERTS / 32) sh.ebits[lane] = 0u;
    __syncwarp();
    for (int q = lane; q < T * k; q += 32) {
        const int e = sh.sel[q / k][q % k];
        atomicOr(&sh.ebits[e >> 5], 1u << (e & 31));
    }
    __syncwarp();
    const int cnt = lane < HFQ_MAX_EXPERTS / 32 ? __popc(sh.ebits[lane]) : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane < HFQ_MAX_EXPERTS / 32) sh.wbase[lane] = incl - cnt;
    const int U = __shfl_sync(0xffffffffu, incl, 31);
    for (int u = lane; u < kMaxU; u += 32) sh.umask[u] = 0u;
    __syncwarp();
    for (int q = lane; q < T * k; q += 32) {
        const int t = q / k, j = q % k, e = sh.sel[t][j];
        const int u = sh.wbase[e >> 5] + __popc(sh.ebits[e >> 5] & ((1u << (e & 31)) - 1u));
        sh.uexp[u] = e;
        sh.ujt[u][t] = (signed char)j;
        atomicOr(&sh.umask[u], 1u << t);
    }
    __syncwarp();
    // expert bases and locations: from the prefetched tables, or one round of loads
    if (a.tab_pref) {
        cp_async_wait_all();
        __syncwarp();
    }
    for (int u = lane; u < U; u += 32) {
        const int e = sh.uexp[u];
        if (a.tab_pref) {
            sh.ubase[u] = reinterpret_cast<const uint8_t *const *>(tab)[e];
            sh.uloc[u] = a.eloc[l] ? tab[(size_t)a.E * 8 + e] : 0;
        } else {
            sh.ubase[u] = static_cast<const uint8_t *>(a.eptr[l][e]);
            sh.uloc[u] = a.eloc[l] ? a.eloc[l][e] : 0;
        }
    }
    // pairs: lane u (then u + 32) writes expert u's pairs at its prefix offset
    int run = 0;
    for (int u0 = 0; u0 < kMaxU; u0 += 32) {
        const int u = u0 + lane;
        const int n = u < U ? __popc(sh.umask[u]) : 0;
        int inc = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        int q = run + inc - n;
        if (u < U) {
            sh.pair0[u] = q;
            for (unsigned m = sh.umask[u]; m; m &= m - 1u, ++q) {
                const int t = __ffs(m) - 1, j = sh.ujt[u][t];
                sh.pt[q] = t;
                sh.prow[q] = t * k + j;
                sh.pw[q] = sh.wsel[t][j];
            }
        }
        run += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {
        sh.pair0[U] = run;
        sh.U = U;
        sh.P = run;
    }
    __syncwarp();
}

// kFull: host-mapped experts, given routing, the debug timeline or the test
// hook are possible; the other instantiation leaves those paths out (smaller
// code: fewer instruction-cache misses).
template <bool kFull>
__global__ void __launch_bounds__(kThr, 1) verify_kernel(const __grid_constant__ VArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const int H = a.H, I = a.I, k = a.k, T = a.T, NS = a.NS;
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
    const int up_off = (sg.len + 127) / 128 * 128;      // up span's offset within a stage

    uint8_t *ring = smem;
    uint32_t *xp = reinterpret_cast<uint32_t *>(smem + a.xp_off);     // [T][nbH*4][kPiece]
    float *xres = reinterpret_cast<float *>(smem + a.xres_off);       // [T][kMaxDRows]
    float *ysh = reinterpret_cast<float *>(smem + a.ysh_off);         // [kCW][T][kMaxDRows]
    float *hst = reinterpret_cast<float *>(smem + a.hst_off);         // [kCW][2][nbI*4][kHStride]
    VShared &sh = *reinterpret_cast<VShared *>(smem + a.sh_off);
    uint8_t *tab = smem + a.tab_off;                                   // [E] u64 expert table, [E] u8 locations
    const WaitCtx wc{a.ctl, a.timeout_ns, &sh.abort};

    if (tid == 0) {
        for (int s = 0; s < kMaxNS; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], kCW);
            sh.armed_seq[s] = -1;
        }
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && a.tab_pref) fetch_tables(a, 0, tab);
    __syncthreads();

    int stage_base = 0;                 // ring items of earlier layers (same in every warp)
    for (int l = 0; l < a.L; ++l) {
        vstamp<kFull>(a, l, 0, tid == 0);
        // ---------------------------------------------- 1. route, pairs, inputs
        if (warp < T) {
            if (kFull && a.idx_in) {
                for (int j = lane; j < k; j += 32) {
                    int e = a.idx_in[warp * k + j];
                    if ((unsigned)e >= (unsigned)a.E) {
                        // a caller's id outside [0, E): recorded; expert 0 stands
                        // in so that every table index stays in range
                        atomicCAS(a.ctl, 0u, (unsigned)HFQ_ERR_ARG);
                        e = 0;
                    }
                    sh.sel[warp][j] = e;
                    sh.wsel[warp][j] = a.wts_in[warp * k + j];
                }
            } else {
                int e;
                float w;
                warp_route(a.logits + ((size_t)l * T + warp) * a.E, a.E, k, e, w);
                if (lane < k) {
                    if ((unsigned)e >= (unsigned)a.E) {
                        atomicCAS(a.ctl, 0u, (unsigned)HFQ_ERR_ARG);
                        sh.abort = 1;
                        e = 0;
                    }
                    sh.sel[warp][lane] = e;
                    sh.wsel[warp][lane] = w;
                }
            }
        }
        {
            // layer input: token t, values 8*tid .. 8*tid+7 (Hp/8 <= 256 groups)
            const uint16_t *xin = l == 0 ? a.x0 : a.xbuf + (size_t)(l & 1) * T * H;
            uint4 xq[kMaxT];                      // every token's 8 values in flight at once
#pragma unroll
            for (int t = 0; t < kMaxT; ++t)
                xq[t] = (t < T && warp < kCW && 8 * tid < H)
                            ? __ldcg(reinterpret_cast<const uint4 *>(xin + (size_t)t * H) + tid)
                            : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int t = 0; t < kMaxT; ++t) {
                if (t >= T || warp >= kCW) break;
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0.0f;
                if (8 * tid < H) {
                    const uint4 q = xq[t];
                    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        v[2 * r] = __uint_as_float(w4[r] << 16);
                        v[2 * r + 1] = __uint_as_float(w4[r] & 0xFFFF0000u);
                    }
                }
                if (8 * tid < Hp) build_x_piece(v, xp + ((size_t)t * nbH * 4 + (tid >> 3)) * kPiece);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * tid + i - d_lo;
                    if (r >= 0 && r < n_d) xres[t * kMaxDRows + r] = v[i];
                }
            }
            if (warp < kCW)
                for (int i = tid; i < kCW * T * kMaxDRows; i += kCW * 32) ysh[i] = 0.0f;
        }
        __syncthreads();
        vstamp<kFull>(a, l, 1, tid == 0);
        if (warp == 0) build_pairs(sh, a, l, tab);
        if (__syncthreads_or(sh.abort)) break;
        vstamp<kFull>(a, l, 2, tid == 0);
        const int U = sh.U, P = sh.P;
        if (a.idx_all && c == 0 && warp < T && lane < k) {
            a.idx_all[((size_t)l * T + warp) * k + lane] = sh.sel[warp][lane];
            a.wts_all[((size_t)l * T + warp) * k + lane] = sh.wsel[warp][lane];
        }

        if (warp >= kCW) {
            // ------------------------------------------ 2. producer warps
            for (int i = 0; i < 2 * U && !sh.abort; ++i) {
                const int seq = stage_base + i, s = seq % NS, u = i < U ? i : i - U;
                // a stage always has the same producer: its uses are armed in order
                if (s % kPW != warp - kCW) continue;
                if (seq >= NS) {
                    int ok = 1;
                    if (lane == 0) {
                        ok = wait_mbar_phase(wc, &sh.empty[s], ((seq / NS) - 1) & 1) ? 1 : 0;
                        note_wait(a, ok, 1, l, seq);
                    }
                    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                }
                // the stage's last readers released it through the empty barrier,
                // which this wait acquired: the bulk copy may overwrite it
                const uint8_t *base = sh.ubase[u];
                if (((uintptr_t)base & 15u) != 0) {               // bulk copies start on 16 bytes
                    if (lane == 0) { atomicCAS(a.ctl, 0u, (unsigned)HFQ_ERR_ARG); sh.abort = 1; }
                    break;
                }
                uint8_t *st = ring + (size_t)s * a.stage_bytes;
                if (lane == 0) {
                    sh.armed_seq[s] = seq;
                    // consumer warps with no pair in this item do not touch the
                    // stage: release it for them in this use's phase (pairs of an
                    // item are contiguous and go to warps p mod kCW)
                    const int np = min(kCW, sh.pair0[u + 1] - sh.pair0[u]);
                    if (np < kCW) mbar_arrive_cnt(&sh.empty[s], (uint32_t)(kCW - np));
                }
                if (!(kFull && sh.uloc[u])) {
                    if (lane == 0) {
                        // expert bytes are read once per step: evict them first from L2
                        const uint64_t pol = l2_evict_first_policy();
                        if (i < U) {
                            mbar_arrive_expect_tx(&sh.full[s], (uint32_t)(sg.len + su.len));
                            if (sg.len) bulk_g2s_hint(st, base + sg.src, (uint32_t)sg.len, &sh.full[s], pol);
                            if (su.len) bulk_g2s_hint(st + up_off, base + su.src, (uint32_t)su.len, &sh.full[s], pol);
                        } else {
                            mbar_arrive_expect_tx(&sh.full[s], (uint32_t)sd.len);
                            if (sd.len) bulk_g2s_hint(st, base + sd.src, (uint32_t)sd.len, &sh.full[s], pol);
                        }
                    }
                } else {
                    // host-mapped expert: 16-byte loads over PCIe, four in flight per lane
                    const int nsp = i < U ? 2 : 1;
                    for (int sp = 0; sp < nsp; ++sp) {
                        const Span &S = i < U ? (sp ? su : sg) : sd;
                        uint8_t *dst = st + (sp ? up_off : 0);
                        for (int o = lane * 16; o < S.len; o += 32 * 16 * 4) {
                            uint4 v[4];
#pragma unroll
                            for (int r = 0; r < 4; ++r)
                                if (o + r * 512 < S.len) v[r] = ld_nc_v4(base + S.src + o + r * 512);
#pragma unroll
                            for (int r = 0; r < 4; ++r)
                                if (o + r * 512 < S.len) *reinterpret_cast<uint4 *>(dst + o + r * 512) = v[r];
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.full[s]);
                }
                vstamp<kFull>(a, l, 8, lane == 0 && i == U - 1);
                vstamp<kFull>(a, l, 10 + i, lane == 0 && i < 10);
            }
            vstamp<kFull>(a, l, 9, lane == 0 && warp == kCW);
        } else {
            // ------------------------------------------ 3. gate/up items
            const int pb = lane >> 2, pq = lane & 3;
            const bool has_piece = pb < nbH;
            bool ok = true;
            for (int u = 0; u < U; ++u) {
                const int seq = stage_base + u, s = seq % NS;
                const uint8_t *st = ring + (size_t)s * a.stage_bytes;
                int p = sh.pair0[u] + ((warp - sh.pair0[u]) % kCW + kCW) % kCW;
                // items without a pair of this warp are skipped: the producer
                // released the stage for this warp when it armed the item
                if (p >= sh.pair0[u + 1]) continue;
                if (ok) {
                    int w = 1;
                    if (lane == 0) {
                        // this use armed first: the full barrier's earlier uses
                        // are then complete and the parity names this use alone
                        w = (wait_armed(wc, &sh.armed_seq[s], seq) &&
                             wait_mbar_phase(wc, &sh.full[s], (seq / NS) & 1)) ? 1 : 0;
                        note_wait(a, w, 2, l, seq);
                    }
                    ok = __shfl_sync(0xffffffffu, w, 0) != 0;
                    vstamp<kFull>(a, l, 3, lane == 0 && u == 0 && warp == 0);
                }
                for (; p < sh.pair0[u + 1] && ok; p += kCW) {
                    uint32_t X[32];
                    int xe = 0;
                    float sxp = 0.0f;
                    if (has_piece) {
                        const uint32_t *pc = xp + ((size_t)sh.pt[p] * nbH * 4 + lane) * kPiece;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint4 q = reinterpret_cast<const uint4 *>(pc)[i];
                            X[4 * i] = q.x; X[4 * i + 1] = q.y; X[4 * i + 2] = q.z; X[4 * i + 3] = q.w;
                        }
                        const uint2 es = *reinterpret_cast<const uint2 *>(pc + 32);
                        xe = (int)es.x;
                        sxp = __uint_as_float(es.y);
                    }
                    vstamp<kFull>(a, l, 24, lane == 0 && warp == 0 && p == 0);
                    float *hrow = a.h + (size_t)sh.prow[p] * Ip + gu_lo;
                    const uint8_t *g0 = st + sg.delta, *u0 = st + up_off + su.delta;
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
                                const uint2 w = live[i] ? *reinterpret_cast<const uint2 *>(pw[i] + 8 * wq)
                                                        : make_uint2(0u, 0u);
                                acc[i] = nib8_dot_bf16(w.x, X + 8 * wq, acc[i]);
                                acc[i] = nib8_dot_bf16(w.y, X + 8 * wq + 4, acc[i]);
                            }
                        }
                        // partial = zero * sum(x) + scale * sum(q * x) over this lane's 64
                        float v[kD];
#pragma unroll
                        for (int i = 0; i < kD; ++i)
                            v[i] = live[i] ? fmaf(sz[i].x, scale2(acc[i], 133 - xe), sz[i].y * sxp) : 0.f;
                        // lane l: total of value (l >> 2) & 7: gate row (l >> 2) for
                        // l < 16, the matching up row 16 lanes higher
                        const float g = warp_sum_many<2 * kGuRows>(v);
                        const float uu = __shfl_down_sync(0xffffffffu, g, 16);
                        const int i = lane >> 2;
                        if (lane < 16 && (lane & 3) == 0 && r0 + i < n_gu) hrow[r0 + i] = silu(g) * uu;
                    }
                    vstamp<kFull>(a, l, 25, lane == 0 && warp == 0 && p == 0);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.empty[s]);        // this warp is done with the stage
            }
            // ------------------------------------------ 4. h exchange
            unsigned *hcnt = a.ctl + kCtlH + (size_t)l * kCtlHStride;
            consumer_sync();
            vstamp<kFull>(a, l, 4, tid == 0);
            if (tid == 0) {
                if (!ok) sh.abort = 1;
                __threadfence();
                red_release_gpu_add(hcnt, 1u);
                if (!sh.abort && !wait_counter_ge(wc, hcnt, (unsigned)G)) {
                    sh.abort = 1;
                    note_wait(a, false, 3, l, 0);
                }
            }
            consumer_sync();
            vstamp<kFull>(a, l, 5, tid == 0);
            ok = ok && !sh.abort;

            // ------------------------------------------ 5. down items
            // Lane: piece pc (64 values of h) of row rs of each pass; Pl lanes
            // per row, 32 / Pl rows per pass.  The warp's pairs in order; the
            // next pair's h is copied (cp.async) into the other staging buffer
            // while the current pair computes.
            const int Pl = nbI * 4, RP = 32 / Pl;
            const int pc = lane % Pl, rs = lane / Pl;
            float *hw0 = hst + (size_t)warp * 2 * Pl * kHStride;      // two buffers per warp
            auto stage_h = [&](int p, float *hw) {
                if (p < P) {
                    const float *src = a.h + (size_t)sh.prow[p] * Ip;
                    for (int i = lane; i < Ip / 4; i += 32) {
                        float *dst = hw + (i >> 4) * kHStride + (i & 15) * 4;
                        if (4 * i < I) cp_async16(dst, src + 4 * i);
                        else *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
                cp_async_commit();                     // one group per call, empty or not
            };
            int pnext = warp, buf = 0;                 // this warp's next pair, its buffer
            stage_h(pnext, hw0);
            for (int u = 0; u < U; ++u) {
                const int seq = stage_base + U + u, s = seq % NS;
                const uint8_t *st = ring + (size_t)s * a.stage_bytes;
                bool waited = false;
                // no pair of this warp in the item: skipped (released by the producer)
                if (pnext >= sh.pair0[u + 1]) continue;
                while (ok && pnext < sh.pair0[u + 1]) {
                    const int p = pnext;
                    float *hw = hw0 + (size_t)buf * Pl * kHStride;
                    pnext += kCW;
                    buf ^= 1;
                    __syncwarp();                      // the other buffer's last reader is done
                    stage_h(pnext, hw0 + (size_t)buf * Pl * kHStride);
                    cp_async_wait_group1();            // this pair's group has landed
                    __syncwarp();
                    float2 hr[32];
                    float2 hs2 = make_float2(0.f, 0.f);
                    {
                        const float4 *hp = reinterpret_cast<const float4 *>(hw + pc * kHStride);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float4 q = hp[i];
                            hr[2 * i] = make_float2(q.x, q.y);
                            hr[2 * i + 1] = make_float2(q.z, q.w);
                            hs2.x += q.x + q.z;
                            hs2.y += q.y + q.w;
                        }
                    }
                    if (!waited) {
                        int w = 1;
                        if (lane == 0) {
                            w = (wait_armed(wc, &sh.armed_seq[s], seq) &&
                                 wait_mbar_phase(wc, &sh.full[s], (seq / NS) & 1)) ? 1 : 0;
                            note_wait(a, w, 4, l, seq);
                        }
                        ok = __shfl_sync(0xffffffffu, w, 0) != 0;
                        waited = true;
                        if (!ok) break;
                    }
                    vstamp<kFull>(a, l, 26, lane == 0 && warp == 0 && p == 0);
                    const uint8_t *d0 = st + sd.delta + (pc >> 2) * kBlockBytes;   // this lane's block of each row
                    const float wp = sh.pw[p];
                    float *yt = ysh + ((size_t)warp * T + sh.pt[p]) * kMaxDRows;
#pragma unroll 1
                    for (int p0 = 0; p0 * RP < n_d; p0 += 4) {      // four passes side by side
                        // rows past n_d repeat the last row (inside the span; their
                        // sums are dropped) so the four passes run side by side
                        // without a branch
                        float v[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int ri = min((p0 + q) * RP + rs, n_d - 1);
                            const uint8_t *blk = d0 + (size_t)ri * rowB_d;
                            const float2 sz = *reinterpret_cast<const float2 *>(blk);
                            uint32_t wv[8];
                            lds_words(blk + 8 + (pc & 3) * 32, wv);
                            v[q] = finish_dot(nib64_fma(wv, hr), hs2, sz.x, sz.y);
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            for (int o = Pl >> 1; o > 0; o >>= 1) v[q] += __shfl_xor_sync(0xffffffffu, v[q], o);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int ri = (p0 + q) * RP + rs;
                            if (pc == 0 && ri < n_d) yt[ri] += wp * v[q];
                        }
                    }
                    vstamp<kFull>(a, l, 27, lane == 0 && warp == 0 && p == 0);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.empty[s]);
            }
            cp_async_wait_all();
            if (!ok) sh.abort = 1;
            // the next layer's tables travel while the other warps finish
            if (warp == 0 && a.tab_pref && l + 1 < a.L) fetch_tables(a, l + 1, tab);
        }
        stage_base += 2 * U;
        __syncthreads();
        vstamp<kFull>(a, l, 6, tid == 0);

        // ---------------------------------------------- 6. combine, residual
        if (!sh.abort && tid < T * n_d) {
            const int t = tid / n_d, ri = tid - t * n_d, r = d_lo + ri;
            float y = 0.0f;
#pragma unroll
            for (int w = 0; w < kCW; ++w) y += ysh[((size_t)w * T + t) * kMaxDRows + ri];
            const bool last = l == a.L - 1;
            const size_t o = (size_t)t * H + r;
            if (a.y) a.y[(size_t)l * T * H + o] = y;
            if (a.y_bf16 && last) a.y_bf16[o] = float_to_bf16_bits(y);
            uint16_t *xo = last ? a.x_out : (a.xbuf ? a.xbuf + (size_t)((l + 1) & 1) * T * H : nullptr);
            if (xo) xo[o] = float_to_bf16_bits(xres[t * kMaxDRows + ri] + y);
        }
        vstamp<kFull>(a, l, 7, tid == 0);
        if (l + 1 < a.L) {
            __syncthreads();
            if (tid == 0) {
                unsigned *bar = a.ctl + kCtlBar + l;
                __threadfence();
                red_release_gpu_add(bar, 1u);
                if (!sh.abort && !wait_counter_ge(wc, bar, (unsigned)(G + (kFull ? a.extra_arrivals : 0)))) {
                    sh.abort = 1;
                    note_wait(a, false, 5, l, 0);
                }
            }
            if (__syncthreads_or(sh.abort)) break;
        }
    }

    // no copy may still be writing this CTA's shared memory when it exits:
    // the tables' cp.async group, and every stage's last armed phase (bounded)
    cp_async_wait_all();
    __syncthreads();
    if (tid < NS) {
        const int seq = sh.armed_seq[tid];
        if (seq >= 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&sh.full[tid], (seq / NS) & 1) && !deadline_passed(t0, a.timeout_ns)) {
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

inline size_t up128(size_t b) { return (b + 127) / 128 * 128; }

}  // namespace

// 2..8 tokens through verify_kernel.  HFQ_ERR_UNSUPPORTED (no message, no
// launch) for a shape or alignment this kernel does not take.
hfq_status verify_launch(const hfq4_layer *layers, int L, const float *logits, const int32_t *idx_in,
                         const float *wts_in, const void *x0, bool x0_f32, int T, int k, uint16_t *x_out,
                         uint16_t *xbuf, float *h, float *y, uint16_t *y_bf16, int32_t *idx_all,
                         float *wts_all, unsigned *ctl, long long timeout_ns, int extra_arrivals,
                         cudaStream_t s)
{
    const int H = layers[0].hidden, I = layers[0].inter, E = layers[0].n_experts;
    const int G = sm_count();
    if (G <= 0) return fail(HFQ_ERR_CUDA, "no CUDA device");
    if (L < 1 || L > HFQ_MAX_STACK_LAYERS || T < 2 || T > kMaxT || k < 1 || T * k > kMaxP)
        return HFQ_ERR_UNSUPPORTED;
    if (x0_f32 || expert_bytes(H, I) % 16) return HFQ_ERR_UNSUPPORTED;
    const int nbH = (H + kBlock - 1) / kBlock, nbI = (I + kBlock - 1) / kBlock;
    if (nbI != 1 && nbI != 2 && nbI != 4) return HFQ_ERR_UNSUPPORTED;     // 4 nbI lanes per down row
    if (H > kBlock * 8 || H % 8 || I > kBlock * 4 || I % 16 || E > HFQ_MAX_EXPERTS) return HFQ_ERR_UNSUPPORTED;
    if ((H + G - 1) / G > kMaxDRows || (L > 1 && !xbuf) || !aligned16(x0) || (xbuf && !aligned16(xbuf)) ||
        !aligned16(h))
        return HFQ_ERR_UNSUPPORTED;

    VArgs a;
    memset(&a, 0, sizeof a);
    for (int l = 0; l < L; ++l) {
        a.eptr[l] = layers[l].expert_ptr;
        a.eloc[l] = layers[l].expert_loc;
    }
    a.logits = logits; a.idx_in = idx_in; a.wts_in = wts_in;
    a.x0 = static_cast<const uint16_t *>(x0); a.x_out = x_out; a.xbuf = xbuf; a.h = h; a.y = y;
    a.y_bf16 = y_bf16; a.idx_all = idx_all; a.wts_all = wts_all;
    a.ctl = ctl; a.timeout_ns = timeout_ns; a.extra_arrivals = extra_arrivals;
    a.timeline = static_cast<unsigned long long *>(option_timeline());
    a.L = L; a.T = T; a.E = E; a.k = k; a.H = H; a.I = I;

    // shared-memory layout: ring stages, then the fixed parts
    const size_t rowB_gu = (size_t)nbH * kBlockBytes, rowB_d = (size_t)nbI * kBlockBytes;
    const size_t gspan = up128((size_t)((I + G - 1) / G) * rowB_gu + 15);
    const size_t dspan = up128((size_t)((H + G - 1) / G) * rowB_d + 15);
    const size_t stage = std::max(2 * gspan, dspan);
    size_t fixed = 0;
    const size_t xp_b = (size_t)T * nbH * 4 * kPiece * 4;
    const size_t xres_b = (size_t)T * kMaxDRows * 4;
    const size_t ysh_b = (size_t)kCW * T * kMaxDRows * 4;
    const size_t hst_b = (size_t)kCW * 2 * nbI * 4 * kHStride * 4;
    const size_t tab_b = up128((size_t)E * 9);
    fixed = xp_b + xres_b + ysh_b + hst_b + tab_b + up128(sizeof(VShared));

    // the instantiation for this launch and its shared-memory limit (set once)
    bool full = a.timeline != nullptr || idx_in != nullptr || extra_arrivals != 0;
    for (int l = 0; l < L; ++l) full = full || layers[l].expert_loc != nullptr;
    const void *kernel = full ? (const void *)verify_kernel<true> : (const void *)verify_kernel<false>;
    static int dyn_limits[2] = {0, 0};
    int &dyn_limit = dyn_limits[full ? 1 : 0];
    if (!dyn_limit) {
        int dev = 0, optin = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "verify kernel attributes: %s", cudaGetErrorString(e));
        int lim = optin - (int)fa.sharedSizeBytes;
        if (lim > kSmemOptin) lim = kSmemOptin;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
        if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "verify kernel attribute %d: %s", lim, cudaGetErrorString(e));
        dyn_limit = lim;
    }
    if (fixed + 2 * stage > (size_t)dyn_limit) return HFQ_ERR_UNSUPPORTED;
    const int NS = (int)std::min<size_t>(kMaxNS, ((size_t)dyn_limit - fixed) / stage);
    a.NS = NS;
    a.stage_bytes = (int)stage;
    size_t off = (size_t)NS * stage;
    a.xp_off = (int)off; off += xp_b;
    a.xres_off = (int)off; off += xres_b;
    a.ysh_off = (int)off; off += ysh_b;
    a.hst_off = (int)off; off += hst_b;
    a.tab_off = (int)up128(off); off = (size_t)a.tab_off + tab_b;
    // prefetched tables: 16-byte copies of whole tables
    a.tab_pref = E % 16 == 0;
    for (int l = 0; l < L; ++l)
        if (!aligned16(layers[l].expert_ptr) || (layers[l].expert_loc && !aligned16(layers[l].expert_loc)))
            a.tab_pref = 0;
    a.sh_off = (int)up128(off);
    const size_t smem = (size_t)a.sh_off + sizeof(VShared);
    if (smem > (size_t)dyn_limit) return HFQ_ERR_UNSUPPORTED;
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
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "verify kernel launch: %s", cudaGetErrorString(e));
    return HFQ_OK;
}

}  // namespace hfq
