// tc.cu - the token-batched expert path on the fifth-generation tensor cores
// (tcgen05), for prefill chunks where an expert sees many tokens.
//
// Per expert e with T_e routed (token, slot) pairs (grouped by moe_route):
//   G = X_e Wg^T, U = X_e Wu^T   (bf16 x bf16 -> f32 in tensor memory)
//   H_e = silu(G) * U, kept as two bf16 parts: hi = bf16(H_e), lo = bf16(H_e - hi)
//   O = hi Wd^T + lo Wd^T         (bf16 x bf16 -> f32), one row per pair
// h keeps about 16 significant bits that way: a single bf16 rounding of h
// would not be unique (a value near a rounding boundary goes either way with
// f32 errors of the gate/up sums) and would move y by a bf16 step of h.
//   y[t] = sum_j w_tj * O[pair (t, j)]   (slot order: deterministic)
// The weights are dequantised from HFQ4 straight into shared memory as bf16,
// RN_bf16(fmaf(scale, q, zero)), in the canonical K-major no-swizzle layout
// the MMA reads (8-row x 16-byte core matrices).  Prior art on the pages: the
// gfx1151 engine README's self-written matrix-core GEMM for prefill
// ("Windows" section); the Strata report, section "three counter-intuitive
// conclusions": prefill is compute-bound, decode bandwidth-bound.
#include <cuda.h>

#include "device.cuh"
#include "ptx.cuh"

namespace hfq {
namespace {

constexpr int kM = 128;                    // weight rows per tile (MMA M)
constexpr int kN = 128;                    // token pairs per tile (MMA N)
constexpr int kKC = 64;                    // K per stage (4 MMAs of K = 16 per matrix)
constexpr int kDqW = 16;                   // dequantising warps
constexpr int kDqThr = kDqW * 32;
constexpr int kMmaWarp = kDqW;             // issues the MMAs
constexpr int kBWarp = kDqW + 1;           // TMA loads of the activation tiles
constexpr int kRawWarp = kDqW + 2;         // TMA loads of the raw HFQ4 bytes
constexpr int kTcThr = (kDqW + 3) * 32;
constexpr int kTileBytes = kM * kKC * 2;   // one 128 x kKC bf16 operand tile (16 KB)
constexpr int kRawW = 144;                 // staged bytes per weight row and HFQ4 block (16-byte window)
constexpr int kMaxTcCtas = 256;            // grid cap (one CTA per SM); sizes the tensor-map slots

// One phase's buffers.  Shared memory: a ring of activation B tiles (TMA,
// 128-byte swizzle) and two raw buffers, each the 144-byte window around one
// HFQ4 block of every weight row of the item.  Tensor memory: the f32
// accumulators (gate [+ up]: kN columns each) and kAStages dequantised A
// stages (weight row m in lane m, two bf16 of K per column), which the MMAs
// read in place: the weights never pass through shared memory, whose
// bandwidth bounds the stage otherwise.
template <bool GU>
struct TcCfg {
    static constexpr int kRows = GU ? 2 * kM : kM;        // weight rows per item (gate rows, then up rows)
    static constexpr int kAStages = 4;                     // dequantised A stages in tensor memory
    static constexpr int kACols = (GU ? 2 : 1) * (kKC / 2);   // TMEM columns of one A stage
    static constexpr int kAccCols = (GU ? 2 : 1) * kN;        // accumulator columns
    static constexpr uint32_t kTmemCols = GU ? 512 : 256;
    static constexpr int kBStages = GU ? 6 : 4;
    static constexpr int kBTiles = GU ? 1 : 2;            // B tiles per stage: x, or h's hi and lo parts
    static constexpr int kBStageBytes = kBTiles * kTileBytes;
    static constexpr int kRawBytes = kRows * kRawW;
    static constexpr int kBOff = 0;
    static constexpr int kRawOff = kBOff + kBStages * kBStageBytes;
    static constexpr int kSmem = kRawOff + 2 * kRawBytes;
    static constexpr int kDqK = GU ? 32 : 16;             // K elements a thread dequantises per stage
    static_assert(kRows * kKC == kDqThr * kDqK, "one dequantisation task per thread and stage");
    static_assert(kAccCols + kAStages * kACols <= (int)kTmemCols, "tensor memory columns");
    static_assert(kAStages <= kBStages, "an A stage's release (the MMA commit of its stage) must still be "
                                        "the barrier phase a dequantising warp can wait on");
};
static_assert(TcCfg<true>::kSmem <= 227 * 1024 - 2048 && TcCfg<false>::kSmem <= 227 * 1024 - 2048,
              "shared memory of the tensor-core kernels");

struct TcArgs {
    const void *const *eptr;       // [E] expert base addresses
    const uint8_t *eloc;           // [E] 0 = HBM, 1 = host-mapped, or null
    const int32_t *cnt, *off, *perm;
    uint16_t *hout;                // gate/up: H_perm out, [pairs][2 I]: hi parts, then lo parts
    float *o;                      // down: O [T*k][H] f32, row q = pair perm[q]
    const int32_t *item_off;       // [E+1] prefix of work items of this phase
    uint8_t *maps;                 // [CTAs][2][128] per-CTA tensor maps of the raw bytes (global)
    unsigned *status;
    long long timeout_ns;
    unsigned long long *timeline;  // debug: [2 phases][64 stages][8] %globaltimer stamps of CTA 0, or null
    int E, H, I, k;
};

constexpr int kTlStages = 64;

// Debug timeline of CTA 0: stamp `s` of its stage c (first 64 stages).
template <bool kOn>
__device__ __forceinline__ void tl_stamp(const TcArgs &a, bool gu, int c, int s)
{
    if (kOn && a.timeline && blockIdx.x == 0 && c < kTlStages)
        a.timeline[((gu ? 0 : 1) * kTlStages + c) * 8 + s] = globaltimer_ns();
}

// Two f32 in one 64-bit register (low word first) and back.
__device__ __forceinline__ unsigned long long f32x2(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ unsigned long long u32x2(uint32_t lo, uint32_t hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

// 8 nibbles -> 8 bf16 weights RN_bf16(fmaf(scale, q, zero)), elements in order.
// The packed two-wide f32 add and FMA of sm_100 round each lane like their
// scalar forms, so the weights are the same bits as with scalar fmaf.
__device__ __forceinline__ uint4 deq8(uint32_t w, float scale, float zero)
{
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    const unsigned long long off = f32x2(-8388608.0f, -8388608.0f);
    const unsigned long long sc = f32x2(scale, scale), ze = f32x2(zero, zero);
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // 0x4B0000qq = 2^23 + q exactly; subtracting 2^23 is exact
        const uint32_t qe = __byte_perm(lo, 0x4B000000u, 0x7440u | j);
        const uint32_t qo = __byte_perm(hi, 0x4B000000u, 0x7440u | j);
        unsigned long long q2;
        asm("add.rn.f32x2 %0, %1, %2;" : "=l"(q2) : "l"(u32x2(qe, qo)), "l"(off));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q2) : "l"(sc), "l"(q2), "l"(ze));
        float fe, fo;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(fe), "=f"(fo) : "l"(q2));
        const __nv_bfloat162 b = __floats2bfloat162_rn(fe, fo);
        r[j] = *reinterpret_cast<const uint32_t *>(&b);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// Bounded wait for the phase of `bar` with the given parity.  Gives up when
// another thread of the CTA has given up (*abort set) or at the deadline, when
// it records HFQ_ERR_TIMEOUT and sets *abort.
__device__ bool tc_wait(const TcArgs &a, uint64_t *bar, uint32_t parity, volatile int *abort)
{
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if (it == 64) t0 = globaltimer_ns();
        if (it > 64 && (it & 15) == 0 && (long long)(globaltimer_ns() - t0) > a.timeout_ns) {
            if (abort) *abort = 1;
            atomicCAS(a.status, 0u, (unsigned)HFQ_ERR_TIMEOUT);
            return false;
        }
    }
}

// First byte of the 16-byte aligned 144-byte window around block b of a row
// (rows are a whole, even number of blocks long, so the window stays inside
// the row): an even block starts on 16 bytes, an odd one 8 bytes past.
__device__ __forceinline__ int raw_window(int b) { return kBlockBytes * b - 8 * (b & 1); }

// One persistent CTA per SM walks the work items (expert, row tile, token
// tile) in K stages of 64.  Warp roles:
//   raw warp   - per HFQ4 block of K, one 3-D TMA load of the 144-byte windows
//                of all the item's weight rows (gate and up) into one of two
//                raw buffers, through this CTA's copy of the raw tensor map,
//                re-targeted to the item's expert (tensormap.replace)
//   B warp     - per stage, one 2-D TMA load of the 128 x 64 activation tile
//                (pair-ordered, 128-byte swizzle) into a ring of B tiles
//   16 warps   - per stage, dequantise a K slice of one weight row each (the
//                row is the thread's TMEM lane) from the raw buffer into one of
//                kAStages A stages in tensor memory (tcgen05.st); the item's
//                epilogue
//   MMA warp   - per stage, the MMAs of the A stage (tensor memory) against
//                the B tile (shared memory)
// Barriers (mbarriers): fullR/rfree per raw buffer, fullB/done per B tile,
// aready per A stage, tfree for the accumulators.  done[s] also frees the A
// stage of its stage.
// kFull: host-mapped experts or the debug timeline are possible; the other
// instantiation leaves those paths out (smaller code, fewer instruction-cache
// misses: about 4 % of a prefill step).
template <bool GU, bool kFull>
__global__ void __launch_bounds__(kTcThr, 1)
    tc_kernel(const __grid_constant__ TcArgs a, const __grid_constant__ CUtensorMap bmap,
              const __grid_constant__ CUtensorMap rmap)
{
    using C = TcCfg<GU>;
    constexpr int RB = C::kBStages;
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int NA = C::kAStages;
    __shared__ uint64_t fullB[RB], done_bar[RB], fullR[2], rfree[2], aready_bar[NA], tfree_bar, fin_bar;
    __shared__ alignas(128) uint8_t s_map[128];
    __shared__ uint32_t tmem_slot;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = GU ? a.H : a.I, Rr = GU ? a.I : a.H;
    const int rtiles = Rr / kM, nK = K / kKC;
    const int rowB = (K + kBlock - 1) / kBlock * kBlockBytes;
    const size_t mg = (size_t)a.I * ((a.H + kBlock - 1) / kBlock) * kBlockBytes;
    const int total = a.item_off[a.E];
    const int my_items = total > (int)blockIdx.x ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int nchunks = my_items * nK;
    volatile int *abortp = &s_abort;

    if (warp == 0) {
        tmem_alloc(&tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < RB; ++s) {
            mbar_init(&fullB[s], 1);
            mbar_init(&done_bar[s], 1);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(&fullR[q], 1);
            mbar_init(&rfree[q], kDqW);
        }
        for (int q = 0; q < NA; ++q) mbar_init(&aready_bar[q], kDqW);
        mbar_init(&tfree_bar, kDqW);
        mbar_init(&fin_bar, 1);
        // the swizzled B tiles need a 1024-byte aligned base
        s_abort = (smem_u32(smem) & 1023u) ? 1 : 0;
        if (s_abort) atomicCAS(a.status, 0u, (unsigned)HFQ_ERR_CUDA);
        fence_mbar_init();
    }
    if (warp == kRawWarp)   // this CTA's template of the raw tensor map
        reinterpret_cast<uint32_t *>(s_map)[lane] = reinterpret_cast<const uint32_t *>(&rmap)[lane];
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_slot;
    uint8_t *const bbuf = smem + C::kBOff;
    uint8_t *const rbuf = smem + C::kRawOff;

    // item -> (expert, first pair, valid pairs, first weight row)
    struct Item {
        int e, p0, nvalid, r0;
    };
    auto item_of = [&](int item) {
        int lo = 0, hi = a.E;                        // item_off[lo] <= item < item_off[lo + 1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (a.item_off[mid] <= item) lo = mid; else hi = mid;
        }
        const int local = item - a.item_off[lo];
        const int rt = local % rtiles, nt = local / rtiles;
        Item t;
        t.e = lo;
        t.p0 = a.off[lo] + nt * kN;
        t.nvalid = min(kN, a.cnt[lo] - nt * kN);
        t.r0 = rt * kM;
        return t;
    };
    const int nb = (K + kBlock - 1) / kBlock;        // HFQ4 blocks (raw loads) per item

    int issued = 0;
    if (s_abort) {
        // nothing runs
    } else if (warp == kRawWarp) {
        // ------------------------------------------------ raw HFQ4 bytes
        uint8_t *gmap = a.maps + (size_t)blockIdx.x * 256;
        int gs = 0;
        for (int it = 0; it < my_items && !*abortp; ++it) {
            const Item t = item_of((int)blockIdx.x + it * (int)gridDim.x);
            const uint8_t *base = static_cast<const uint8_t *>(a.eptr[t.e]) + (GU ? 0 : 2 * mg);
            const bool host = kFull && a.eloc && a.eloc[t.e];
            uint8_t *slot = gmap + (it & 1) * 128;
            if (!host) {
                if (lane == 0) tmap_replace_address(s_map, base);
                __syncwarp();
                tmap_copy_release(slot, s_map);
                if (lane == 0) tmap_acquire(slot);
            }
            for (int b = 0; b < nb && !*abortp; ++b, ++gs) {
                const int q = gs & 1;
                if (gs >= 2 && !tc_wait(a, &rfree[q], (uint32_t)((gs >> 1) - 1) & 1u, abortp)) break;
                uint8_t *dst = rbuf + q * C::kRawBytes;
                if (!host) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&fullR[q], (uint32_t)C::kRawBytes);
                        if (GU) tma_load_3d(dst, slot, raw_window(b), t.r0, 0, &fullR[q]);
                        else tma_load_2d(dst, slot, raw_window(b), t.r0, &fullR[q]);
                    }
                } else {
                    // host-mapped expert: plain 16-byte loads over PCIe
                    for (int i = lane; i < C::kRows * (kRawW / 16); i += 32) {
                        const int row = i / (kRawW / 16), piece = i - row * (kRawW / 16);
                        const uint8_t *src = base + (GU && row >= kM ? mg : 0) +
                                             (size_t)(t.r0 + (row & (kM - 1))) * rowB + raw_window(b) + 16 * piece;
                        *reinterpret_cast<uint4 *>(dst + row * kRawW + 16 * piece) = __ldcv(reinterpret_cast<const uint4 *>(src));
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&fullR[q]);
                }
            }
        }
        // an aborted CTA still lets its last raw loads land before it ends
        // (each buffer holds at most one load in flight)
        if (lane == 0)
            for (int g = max(0, gs - 2); g < gs; ++g) tc_wait(a, &fullR[g & 1], (uint32_t)(g >> 1) & 1u, nullptr);
    } else if (warp == kBWarp) {
        // ------------------------------------------------ activation tiles
        int p0 = 0, nb_issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int it = c / nK, kc = c - it * nK;
            if (kc == 0) p0 = item_of((int)blockIdx.x + it * (int)gridDim.x).p0;
            if (c >= RB && !tc_wait(a, &done_bar[(c - RB) % RB], (uint32_t)((c - RB) / RB) & 1u, abortp)) break;
            if (lane == 0) {
                uint8_t *bst = bbuf + (c % RB) * C::kBStageBytes;
                mbar_arrive_expect_tx(&fullB[c % RB], (uint32_t)C::kBStageBytes);
                tma_load_2d(bst, &bmap, kc * kKC, p0, &fullB[c % RB]);
                if (!GU)        // lo part of h, I columns further on
                    tma_load_2d(bst + kTileBytes, &bmap, a.I + kc * kKC, p0, &fullB[c % RB]);
            }
            nb_issued = c + 1;
            __syncwarp();
        }
        // an aborted CTA still lets its last activation loads land
        if (lane == 0)
            for (int c = max(0, nb_issued - RB); c < nb_issued; ++c)
                tc_wait(a, &fullB[c % RB], (uint32_t)(c / RB) & 1u, nullptr);
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issue
        const uint32_t idesc = umma_idesc_bf16(kM, kN);
        for (int c = 0; c < nchunks; ++c) {
            const int it = c / nK, kc = c - it * nK;
            if (kc == 0 && it > 0 && !tc_wait(a, &tfree_bar, (uint32_t)(it - 1) & 1u, abortp)) break;
            if (!tc_wait(a, &aready_bar[c % NA], (uint32_t)(c / NA) & 1u, abortp)) break;
            if (!tc_wait(a, &fullB[c % RB], (uint32_t)(c / RB) & 1u, abortp)) break;
            tc_fence_after_sync();
            if (lane == 0) tl_stamp<kFull>(a, GU, c, 5);
            if (lane == 0) {
                // the A stage was written to tensor memory by other threads
                // (tcgen05.st, waited for, fenced) and released by aready
                const uint32_t A = tmem + (uint32_t)(C::kAccCols + (c % NA) * C::kACols);
                const uint8_t *B = bbuf + (c % RB) * C::kBStageBytes;
#pragma unroll
                for (int ks = 0; ks < kKC / 16; ++ks) {
                    const uint64_t bd = umma_desc_sw128(B + 32 * ks);
                    umma_bf16_ts(tmem, A + 8 * ks, bd, idesc, (kc | ks) != 0);
                    if (GU)
                        umma_bf16_ts(tmem + kN, A + kKC / 2 + 8 * ks, bd, idesc, (kc | ks) != 0);
                    else        // the same weights against h's lo part
                        umma_bf16_ts(tmem, A + 8 * ks, umma_desc_sw128(B + kTileBytes + 32 * ks), idesc, true);
                }
                umma_commit(&done_bar[c % RB]);
                tl_stamp<kFull>(a, GU, c, 6);
            }
            ++issued;
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ dequantisation
        // task: weight row 32 (warp % 4) + lane of the item (the thread's TMEM
        // lane; gate/up: of the gate rows for warps 0..3 and 8..11, the up rows
        // for 4..7 and 12..15), K elements kq * kDqK .. + kDqK - 1 of the stage
        const int quarter = warp & 3;
        const int mat = GU ? (warp >> 2) & 1 : 0;
        const int kq = GU ? warp >> 3 : warp >> 2;
        const int drow = mat * kM + 32 * quarter + lane;
        const uint32_t a_lane = tmem + ((uint32_t)(32 * quarter) << 16) +
                                (uint32_t)(C::kAccCols + mat * (kKC / 2) + kq * (C::kDqK / 2));
        int gs = -1;
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int it = c / nK, kc = c - it * nK;
            const int j = kc & 3, b = kc >> 2;
            const bool tl = tid == 0;
            if (tl) tl_stamp<kFull>(a, GU, c, 0);
            if (j == 0) ++gs;                         // the stage opens a new raw buffer (HFQ4 block)
            if (j == 0 && !tc_wait(a, &fullR[gs & 1], (uint32_t)(gs >> 1) & 1u, abortp)) break;
            if (tl) tl_stamp<kFull>(a, GU, c, 1);
            // the MMAs of stage c - NA are done: its A stage is free
            if (c >= NA && !tc_wait(a, &done_bar[(c - NA) % RB], (uint32_t)((c - NA) / RB) & 1u, abortp)) break;
            tc_fence_after_sync();
            if (tl) tl_stamp<kFull>(a, GU, c, 2);
            const uint8_t *raw = rbuf + (gs & 1) * C::kRawBytes + drow * kRawW + 8 * (b & 1);
            const float2 sz = *reinterpret_cast<const float2 *>(raw);
            const uint8_t *pw = raw + 8 + 32 * j + kq * (C::kDqK / 2);
            const uint32_t at = a_lane + (uint32_t)((c % NA) * C::kACols);
            if (GU) {
                uint32_t v[16];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(pw + 8 * h);
                    const uint4 d0 = deq8(w.x, sz.x, sz.y), d1 = deq8(w.y, sz.x, sz.y);
                    v[8 * h + 0] = d0.x; v[8 * h + 1] = d0.y; v[8 * h + 2] = d0.z; v[8 * h + 3] = d0.w;
                    v[8 * h + 4] = d1.x; v[8 * h + 5] = d1.y; v[8 * h + 6] = d1.z; v[8 * h + 7] = d1.w;
                }
                tmem_st16(at, v);
            } else {
                uint32_t v[8];
                const uint2 w = *reinterpret_cast<const uint2 *>(pw);
                const uint4 d0 = deq8(w.x, sz.x, sz.y), d1 = deq8(w.y, sz.x, sz.y);
                v[0] = d0.x; v[1] = d0.y; v[2] = d0.z; v[3] = d0.w;
                v[4] = d1.x; v[5] = d1.y; v[6] = d1.z; v[7] = d1.w;
                tmem_st8(at, v);
            }
            tmem_st_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&aready_bar[c % NA]);
                if (j == 3 || kc == nK - 1) mbar_arrive(&rfree[gs & 1]);   // raw buffer read
            }
            if (tl) tl_stamp<kFull>(a, GU, c, 3);

            if (kc == nK - 1) {
                // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (weight
                // rows), columns (token pairs) 32 (w / 4) .. + 31
                if (!tc_wait(a, &done_bar[c % RB], (uint32_t)(c / RB) & 1u, abortp)) break;
                tc_fence_after_sync();
                const Item t = item_of((int)blockIdx.x + it * (int)gridDim.x);
                const int lg = warp & 3, cgp = warp >> 2;
                const int r = lg * 32 + lane;
                const uint32_t trow = tmem + ((uint32_t)(lg * 32) << 16);
#pragma unroll 1
                for (int col = cgp * 32; col < cgp * 32 + 32; col += 16) {
                    float g[16], u[16];
                    tmem_ld16(trow + col, g);
                    if (GU) tmem_ld16(trow + kN + col, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int n = col + jj;
                        if (n >= t.nvalid) break;
                        const int p = t.p0 + n;
                        if (GU) {
                            const float hv = silu(g[jj]) * u[jj];
                            const uint16_t hi = float_to_bf16_bits(hv);
                            uint16_t *hrow = a.hout + (size_t)p * 2 * a.I + t.r0 + r;
                            hrow[0] = hi;
                            hrow[a.I] = float_to_bf16_bits(hv - bf16_bits_to_float(hi));   // exact difference
                        } else
                            a.o[(size_t)p * a.H + t.r0 + r] = g[jj];
                    }
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tfree_bar);
            }
        }
    }
    // no MMA may still write tensor memory, nor a TMA load shared memory,
    // when the CTA ends
    if (warp == kMmaWarp && lane == 0 && issued > 0) {
        umma_commit(&fin_bar);
        tc_wait(a, &fin_bar, 0u, nullptr);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}

// Work items per expert: ceil(cnt/kN) token tiles x (rows/kM) row tiles, for
// the gate/up phase (rows = I) and the down phase (rows = H); exclusive scans.
// The grouping comes from the caller: unless cnt >= 0, off[0] = 0,
// off[e + 1] = off[e] + cnt[e] and off[E] = P, the status word gets
// HFQ_ERR_ARG and both phases get no items (nothing is read or written).
__global__ void tc_plan_kernel(const int32_t *__restrict__ cnt, const int32_t *__restrict__ off, int E,
                               int I, int H, int P, int32_t *__restrict__ gu_off, int32_t *__restrict__ dn_off,
                               unsigned *status)
{
    __shared__ int s_gu[HFQ_MAX_EXPERTS], s_dn[HFQ_MAX_EXPERTS];
    __shared__ int s_bad;
    if (threadIdx.x == 0) s_bad = (off[0] != 0 || off[E] != P);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int c = cnt[e];
        if (c < 0 || off[e + 1] - off[e] != c) s_bad = 1;
        const int tiles = c > 0 ? (c + kN - 1) / kN : 0;
        s_gu[e] = tiles * (I / kM);
        s_dn[e] = tiles * (H / kM);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool bad = s_bad != 0;
        if (bad) atomicCAS(status, 0u, (unsigned)HFQ_ERR_ARG);
        int a = 0, b = 0;
        for (int e = 0; e < E; ++e) {
            gu_off[e] = a; dn_off[e] = b;
            if (!bad) { a += s_gu[e]; b += s_dn[e]; }
        }
        gu_off[E] = a; dn_off[E] = b;
    }
}

// X_perm[q] = x[token of pair perm[q]] as bf16 (16 bytes per thread step);
// pos[perm[q]] = q.
__global__ void tc_gather_kernel(const void *__restrict__ x, int x_f32, const int32_t *__restrict__ perm,
                                 int P, int k, int H, uint16_t *__restrict__ xp, int32_t *__restrict__ pos,
                                 unsigned *status)
{
    const size_t n8 = (size_t)P * H / 8;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t q = i / (H / 8), c = (i - q * (H / 8)) * 8;
        const int pr = perm[q];
        if ((unsigned)pr >= (unsigned)P) {          // not a pair id: recorded, row left alone
            if (c == 0) atomicCAS(status, 0u, (unsigned)HFQ_ERR_ARG);
            continue;
        }
        if (c == 0) pos[pr] = (int32_t)q;
        const size_t src = (size_t)(pr / k) * H + c;
        uint4 v;
        if (x_f32) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + src));
            const float4 b = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + src) + 1);
            __nv_bfloat162 t;
            t = __floats2bfloat162_rn(a.x, a.y); v.x = *reinterpret_cast<uint32_t *>(&t);
            t = __floats2bfloat162_rn(a.z, a.w); v.y = *reinterpret_cast<uint32_t *>(&t);
            t = __floats2bfloat162_rn(b.x, b.y); v.z = *reinterpret_cast<uint32_t *>(&t);
            t = __floats2bfloat162_rn(b.z, b.w); v.w = *reinterpret_cast<uint32_t *>(&t);
        } else {
            v = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + src));
        }
        *reinterpret_cast<uint4 *>(xp + q * H + c) = v;
    }
}

// y[t][r] = sum over slots j (in order) of w[t*k + j] * O[pos[t*k + j]][r],
// four rows per thread step; optional bf16 copy.
// A pair whose position does not lead back to it (perm was not a permutation
// of the pairs) is recorded as HFQ_ERR_ARG and left out of the sum.
__global__ void tc_combine_kernel(const float *__restrict__ o, const int32_t *__restrict__ pos,
                                  const int32_t *__restrict__ perm, const float *__restrict__ wts, int T,
                                  int k, int H, float *__restrict__ y, uint16_t *__restrict__ yb,
                                  unsigned *status)
{
    const size_t n4 = (size_t)T * H / 4;
    const int P = T * k;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t t = i / (H / 4), c = (i - t * (H / 4)) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const float w = wts[t * k + j];
            const int q = pos[t * k + j];
            if ((unsigned)q >= (unsigned)P || perm[q] != (int)(t * k + j)) {
                if (c == 0) atomicCAS(status, 0u, (unsigned)HFQ_ERR_ARG);
                continue;
            }
            const float4 v = __ldg(reinterpret_cast<const float4 *>(o + (size_t)q * H + c));
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
        *reinterpret_cast<float4 *>(y + t * H + c) = acc;
        if (yb) {
            const uint32_t lo = float_to_bf16_bits(acc.x) | ((uint32_t)float_to_bf16_bits(acc.y) << 16);
            const uint32_t hi = float_to_bf16_bits(acc.z) | ((uint32_t)float_to_bf16_bits(acc.w) << 16);
            *reinterpret_cast<uint2 *>(yb + t * H + c) = make_uint2(lo, hi);
        }
    }
}

int tc_sms()
{
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        n = std::min(n, kMaxTcCtas);
    }
    return n;
}

}  // namespace

size_t tc_workspace_bytes(int T, int k, int H, int I, int E)
{
    const size_t P = (size_t)T * k;
    auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
    return r256(P * H * 2) + r256(P * 2 * I * 2) + 2 * r256((size_t)(E + 1) * 4) + r256(P * H * 4) +
           r256(P * 4) + r256((size_t)kMaxTcCtas * 256);
}

// Rows of whole HFQ4 blocks must be a multiple of 16 bytes (an even number of
// blocks) for the tensor maps of the raw bytes; tiles are 128 rows.
bool tc_supported(int H, int I)
{
    const int nbh = (H + kBlock - 1) / kBlock, nbi = (I + kBlock - 1) / kBlock;
    return H % kM == 0 && I % kM == 0 && nbh % 2 == 0 && nbi % 2 == 0;
}

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn()
{
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    }
    return fn;
}

// bf16 [rows][K] (pair-ordered activations or h): 128 x 64 boxes, 128-byte swizzle.
bool encode_act(CUtensorMap *m, const void *base, int K, size_t rows)
{
    const cuuint64_t dim[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t stride[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kKC, (cuuint32_t)kN}, es[2] = {1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dim, stride, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raw HFQ4 bytes of one expert: gate/up as [2][I][rowB] (up = gate + mg), down
// as [H][rowB]; 144-byte x 128-row boxes (x 2 matrices).  `base` is a
// placeholder: the kernel re-targets a copy of the map to each item's expert.
bool encode_raw(CUtensorMap *m, const void *base, bool gu, int rows, int rowB, size_t mg)
{
    const cuuint64_t dim[3] = {(cuuint64_t)rowB, (cuuint64_t)rows, 2};
    const cuuint64_t stride[2] = {(cuuint64_t)rowB, (cuuint64_t)mg};
    const cuuint32_t box[3] = {(cuuint32_t)kRawW, (cuuint32_t)kM, 2}, es[3] = {1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, gu ? 3 : 2, const_cast<void *>(base), dim, stride, box,
                       es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

hfq_status launch_tc(const hfq4_layer &L, const void *x, bool x_f32, int T, int k, const int32_t *cnt,
                     const int32_t *off, const int32_t *perm, const float *wts, float *y,
                     uint16_t *y_bf16, void *ws, unsigned *status, long long timeout_ns,
                     cudaStream_t s)
{
    const int H = L.hidden, I = L.inter, E = L.n_experts;
    const size_t P = (size_t)T * k;
    auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint16_t *xp = reinterpret_cast<uint16_t *>(w);
    w += r256(P * H * 2);
    uint16_t *hp = reinterpret_cast<uint16_t *>(w);        // [P][2 I]: hi, lo
    w += r256(P * 2 * I * 2);
    int32_t *gu_off = reinterpret_cast<int32_t *>(w);
    w += r256((size_t)(E + 1) * 4);
    int32_t *dn_off = reinterpret_cast<int32_t *>(w);
    w += r256((size_t)(E + 1) * 4);
    float *ob = reinterpret_cast<float *>(w);
    w += r256(P * H * 4);
    int32_t *pos = reinterpret_cast<int32_t *>(w);
    w += r256(P * 4);
    uint8_t *maps = w;

    if (!encode_fn()) return fail(HFQ_ERR_CUDA, "tensor-core path: cuTensorMapEncodeTiled unavailable");
    const int rowB_gu = (H + kBlock - 1) / kBlock * kBlockBytes, rowB_dn = (I + kBlock - 1) / kBlock * kBlockBytes;
    const size_t mg = (size_t)I * rowB_gu;
    CUtensorMap xmap, hmap, rmap_gu, rmap_dn;
    if (!encode_act(&xmap, xp, H, P) || !encode_act(&hmap, hp, 2 * I, P) ||
        !encode_raw(&rmap_gu, maps, true, I, rowB_gu, mg) || !encode_raw(&rmap_dn, maps, false, H, rowB_dn, mg))
        return fail(HFQ_ERR_CUDA, "tensor-core path: tensor map encoding failed (H %d, I %d, pairs %zu)", H, I, P);

    static bool attr = false;
    const int smem_gu = TcCfg<true>::kSmem, smem_dn = TcCfg<false>::kSmem;
    if (!attr) {
        cudaFuncSetAttribute(tc_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_gu);
        cudaFuncSetAttribute(tc_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dn);
        cudaFuncSetAttribute(tc_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_gu);
        cudaFuncSetAttribute(tc_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dn);
        attr = true;
    }
    tc_plan_kernel<<<1, 512, 0, s>>>(cnt, off, E, I, H, (int)P, gu_off, dn_off, status);
    // pair-ordered bf16 activations (the TMA tiles need contiguous rows)
    const size_t n8 = P * H / 8;
    tc_gather_kernel<<<(unsigned)std::min<size_t>((n8 + 255) / 256, (size_t)tc_sms() * 16), 256, 0, s>>>(
        x, x_f32 ? 1 : 0, perm, (int)P, k, H, xp, pos, status);
    TcArgs a;
    a.eptr = L.expert_ptr; a.eloc = L.expert_loc; a.cnt = cnt; a.off = off; a.perm = perm;
    a.maps = maps; a.status = status; a.timeout_ns = timeout_ns; a.E = E; a.H = H; a.I = I; a.k = k;
    a.timeline = static_cast<unsigned long long *>(option_timeline());
    const bool full = a.timeline != nullptr || a.eloc != nullptr;
    a.hout = hp; a.o = nullptr; a.item_off = gu_off;
    if (full) tc_kernel<true, true><<<tc_sms(), kTcThr, smem_gu, s>>>(a, xmap, rmap_gu);
    else tc_kernel<true, false><<<tc_sms(), kTcThr, smem_gu, s>>>(a, xmap, rmap_gu);
    a.hout = nullptr; a.o = ob; a.item_off = dn_off;
    if (full) tc_kernel<false, true><<<tc_sms(), kTcThr, smem_dn, s>>>(a, hmap, rmap_dn);
    else tc_kernel<false, false><<<tc_sms(), kTcThr, smem_dn, s>>>(a, hmap, rmap_dn);
    const size_t n4 = (size_t)T * H / 4;
    tc_combine_kernel<<<(unsigned)std::min<size_t>((n4 + 255) / 256, (size_t)tc_sms() * 16), 256, 0, s>>>(
        ob, pos, perm, wts, T, k, H, y, y_bf16, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "tensor-core path launch: %s", cudaGetErrorString(e));
    return HFQ_OK;
}

}  // namespace hfq
