// tc.cu - the token-batched expert path on the fifth-generation tensor cores
// (tcgen05), for prefill chunks where an expert sees many tokens.
//
// Per expert e with T_e routed (token, slot) pairs (grouped by moe_route):
//   G = X_e Wg^T, U = X_e Wu^T   (bf16 x bf16 -> f32 in tensor memory)
//   H_e = bf16(silu(G) * U)
//   O = H_e Wd^T                  (bf16 x bf16 -> f32), one row per pair
//   y[t] = sum_j w_tj * O[pair (t, j)]   (slot order: deterministic)
// The weights are dequantised from HFQ4 straight into shared memory as bf16,
// RN_bf16(fmaf(scale, q, zero)), in the canonical K-major no-swizzle layout
// the MMA reads (8-row x 16-byte core matrices).  Prior art on the pages: the
// gfx1151 engine README's self-written matrix-core GEMM for prefill
// ("Windows" section); the Strata report, section "three counter-intuitive
// conclusions": prefill is compute-bound, decode bandwidth-bound.
#include "device.cuh"
#include "ptx.cuh"

namespace hfq {
namespace {

constexpr int kM = 128;                    // weight rows per tile (MMA M)
constexpr int kN = 128;                    // token pairs per tile (MMA N)
constexpr int kKC = 128;                   // K per pipeline stage (8 MMAs of K = 16)
constexpr int kQB = kKC / 32;              // 16-byte nibble quarters per row and chunk (4)
constexpr int kTcThr = 512;                // 16 warps
constexpr int kTcW = kTcThr / 32;
constexpr int kTileBytes = kM * kKC * 2;   // one 128 x kKC bf16 operand tile
constexpr uint32_t kLbo = (kM / 8) * 128;  // bytes between 8-element K chunks (2048)
constexpr uint32_t kSbo = 128;             // bytes between 8-row groups
constexpr uint32_t kTmemCols = 256;

struct TcArgs {
    const void *const *eptr;       // [E] expert base addresses
    const int32_t *cnt, *off, *perm;
    const float *wts;              // [T*k] routing weights, flat
    const uint16_t *xin;           // gate/up: X_perm [T*k][H] or x [T][H]; down: H_perm [T*k][I] (bf16)
    int x_direct;                  // gate/up reads row perm[q] / k of x instead of row q of X_perm
    uint16_t *hout;                // gate/up: H_perm out
    float *o;                      // down: O [T*k][H] f32, row q = pair perm[q]
    const int32_t *item_off;       // [E+1] prefix of work items of this phase
    unsigned *status;
    long long timeout_ns;
    int E, H, I, k;
};

// Offset of element (row, kk) of a 128 x 64 operand tile in the canonical layout.
__device__ __forceinline__ uint32_t tile_off(int row, int k8)
{
    return (uint32_t)(row >> 3) * kSbo + (uint32_t)(row & 7) * 16u + (uint32_t)k8 * kLbo;
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

__device__ bool tc_wait(const TcArgs &a, uint64_t *bar, uint32_t parity, int &abort)
{
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (it == 64) t0 = globaltimer_ns();
        if (it > 64 && (it & 15) == 0 && (long long)(globaltimer_ns() - t0) > a.timeout_ns) {
            abort = 1;
            atomicCAS(a.status, 0u, (unsigned)HFQ_ERR_TIMEOUT);
            return false;
        }
    }
}

// One persistent CTA per SM walks the work items (expert, row tile, token tile).
template <bool GU>
__global__ void __launch_bounds__(kTcThr, 1) tc_kernel(const __grid_constant__ TcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int kOps = GU ? 3 : 2;                 // operand tiles per stage (A0 [A1] B)
    __shared__ uint64_t mma_bar[2];
    __shared__ uint32_t tmem_slot;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = GU ? a.H : a.I, R = GU ? a.I : a.H;
    const int rtiles = R / kM, nK = K / kKC;
    const int rowB = (K + kBlock - 1) / kBlock * kBlockBytes;
    const size_t mg = (size_t)a.I * ((a.H + kBlock - 1) / kBlock) * kBlockBytes;
    const uint32_t idesc = umma_idesc_bf16(kM, kN);

    if (warp == 0) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&mma_bar[0], 1);
        mbar_init(&mma_bar[1], 1);
        s_abort = 0;
        fence_mbar_init();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_slot;
    int abort = 0;
    uint32_t commits[2] = {0u, 0u};
    uint32_t chunk = 0;                              // stages used so far (buffer = chunk & 1)
    const int total = a.item_off[a.E];

    // Loads: a warp instruction reads 8 rows x 64 contiguous bytes (4 lanes
    // of 16 bytes per row, rows fastest across lanes), and the 8 lanes of each
    // shared-memory store phase write one 128-byte core-matrix column (8
    // consecutive rows, one K chunk).  Weight rows: rid = (lane & 7) +
    // 8 * (warp + kTcW * i), i < kRI (gate/up: rows >= 128 are the up
    // matrix), quarter qq = lane >> 3.  Activation pieces: token n =
    // (lane & 7) + 8 * (b & 15), K piece 4 * (b >> 4) + qq, b = warp + kTcW * i.
    // The next chunk's loads (of this item or, at its last chunk, of the next
    // item) are in flight while a chunk is dequantised and multiplied.
    constexpr int kRI = (GU ? 2 * kM : kM) / (8 * kTcW);   // weight rows per thread and chunk
    const int qq = lane >> 3, rl = lane & 7;
    struct Geo {
        int p0, nvalid, r0;
        const uint8_t *gbase, *ubase;                // gate (or down) and up matrices
        const uint16_t *xrow;                        // this thread's activation row, or null
    };
    static_assert(kTcW == 16, "one activation row per thread: n = (lane & 7) + 8 * warp");
    const int xn = rl + 8 * warp;
    auto geo_of = [&](int item) {
        int lo = 0, hi = a.E;                        // item_off[lo] <= item < item_off[lo + 1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (a.item_off[mid] <= item) lo = mid; else hi = mid;
        }
        const int e = lo, local = item - a.item_off[e];
        const int rt = local % rtiles, nt = local / rtiles;
        Geo g;
        g.p0 = a.off[e] + nt * kN;
        g.nvalid = min(kN, a.cnt[e] - nt * kN);
        g.r0 = rt * kM;
        const uint8_t *base = static_cast<const uint8_t *>(a.eptr[e]);
        g.gbase = (GU ? base : base + 2 * mg) + (size_t)g.r0 * rowB;
        g.ubase = base + mg + (size_t)g.r0 * rowB;
        g.xrow = nullptr;
        if (xn < g.nvalid) {
            const int q = g.p0 + xn;
            g.xrow = a.xin + (size_t)(GU && a.x_direct ? a.perm[q] / a.k : q) * K;
        }
        return g;
    };
    float2 nsz[kRI];
    uint4 nw[kRI];
    uint4 nx[(kN * kKC / 8) / kTcThr];
    auto load = [&](const Geo &g, int kc2) {
        const int blk = (kc2 * kKC) / kBlock, sub = ((kc2 * kKC) % kBlock) / 2;   // nibble byte
#pragma unroll
        for (int i = 0; i < kRI; ++i) {
            const int rid = rl + 8 * (warp + kTcW * i);
            const uint8_t *rp = (GU && rid >= kM ? g.ubase : g.gbase) + (size_t)(rid & (kM - 1)) * rowB +
                                (size_t)blk * kBlockBytes;
            nsz[i] = __ldg(reinterpret_cast<const float2 *>(rp));
            // the payload of an even block starts at 8 mod 16: two 8-byte loads
            const uint2 lo = __ldg(reinterpret_cast<const uint2 *>(rp + 8 + sub + 16 * qq));
            const uint2 hi = __ldg(reinterpret_cast<const uint2 *>(rp + 16 + sub + 16 * qq));
            nw[i] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
#pragma unroll
        for (int i = 0; i < (kN * kKC / 8) / kTcThr; ++i) {
            const int k8 = 4 * ((warp + kTcW * i) >> 4) + qq;
            nx[i] = g.xrow ? __ldg(reinterpret_cast<const uint4 *>(g.xrow + kc2 * kKC + k8 * 8))
                           : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    Geo cur{};
    if ((int)blockIdx.x < total) {
        cur = geo_of(blockIdx.x);
        load(cur, 0);
    }
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Geo g = cur;
        const int p0 = g.p0, nvalid = g.nvalid, r0 = g.r0;
        const int next = item + (int)gridDim.x;
        Geo ng{};
        if (next < total) ng = geo_of(next);

        for (int kc = 0; kc < nK; ++kc, ++chunk) {
            const int s = chunk & 1;
            uint8_t *st = smem + (size_t)s * kOps * kTileBytes;
            float2 sz[kRI];
            uint4 w[kRI];
            uint4 xv[(kN * kKC / 8) / kTcThr];
#pragma unroll
            for (int i = 0; i < kRI; ++i) { sz[i] = nsz[i]; w[i] = nw[i]; }
#pragma unroll
            for (int i = 0; i < (kN * kKC / 8) / kTcThr; ++i) xv[i] = nx[i];
            if (!abort) {
                if (kc + 1 < nK) load(g, kc + 1);
                else if (next < total) load(ng, 0);
            }
            if (commits[s] && !abort) tc_wait(a, &mma_bar[s], (commits[s] - 1) & 1, abort);
            if (!abort) {
                // weights: row rid, K pieces 4 qq .. 4 qq + 3 of this chunk
#pragma unroll
                for (int i = 0; i < kRI; ++i) {
                    const int rid = rl + 8 * (warp + kTcW * i);
                    uint8_t *dst = st + (GU && rid >= kM ? kTileBytes : 0);
                    const int rr = rid & (kM - 1);
                    *reinterpret_cast<uint4 *>(dst + tile_off(rr, 4 * qq + 0)) = deq8(w[i].x, sz[i].x, sz[i].y);
                    *reinterpret_cast<uint4 *>(dst + tile_off(rr, 4 * qq + 1)) = deq8(w[i].y, sz[i].x, sz[i].y);
                    *reinterpret_cast<uint4 *>(dst + tile_off(rr, 4 * qq + 2)) = deq8(w[i].z, sz[i].x, sz[i].y);
                    *reinterpret_cast<uint4 *>(dst + tile_off(rr, 4 * qq + 3)) = deq8(w[i].w, sz[i].x, sz[i].y);
                }
                // activations: 128 token rows x kKC values, 16 bytes per piece
                uint8_t *bt = st + (size_t)(kOps - 1) * kTileBytes;
#pragma unroll
                for (int i = 0; i < (kN * kKC / 8) / kTcThr; ++i) {
                    const int blkid = warp + kTcW * i;
                    const int n = rl + 8 * (blkid & 15), k8 = 4 * (blkid >> 4) + qq;
                    *reinterpret_cast<uint4 *>(bt + tile_off(n, k8)) = xv[i];
                }
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0 && !abort && !s_abort) {
                tc_fence_after_sync();
                const uint8_t *bt = st + (size_t)(kOps - 1) * kTileBytes;
#pragma unroll
                for (int ks = 0; ks < kKC / 16; ++ks) {
                    const uint64_t bd = umma_desc(bt + 2 * ks * kLbo, kLbo, kSbo);
                    umma_bf16(tmem, umma_desc(st + 2 * ks * kLbo, kLbo, kSbo), bd, idesc,
                              (kc | ks) != 0);
                    if (GU)
                        umma_bf16(tmem + kN, umma_desc(st + kTileBytes + 2 * ks * kLbo, kLbo, kSbo),
                                  bd, idesc, (kc | ks) != 0);
                }
                umma_commit(&mma_bar[s]);
            }
            ++commits[s];
            if (abort && tid == 0) s_abort = 1;
        }
        // all MMAs of the item are complete once its last commit has arrived
        const int sl = (chunk - 1) & 1;
        if (!abort && !s_abort) tc_wait(a, &mma_bar[sl], (commits[sl] - 1) & 1, abort);
        tc_fence_after_sync();
        if (!abort && !s_abort) {
            constexpr int kCols = kN / (kTcW / 4);                // columns per warp
            const int lg = warp & 3, half = warp >> 2;          // TMEM lane group, column group
            const int r = lg * 32 + lane;
            const uint32_t trow = tmem + ((uint32_t)(lg * 32) << 16);
#pragma unroll 1
            for (int c = half * kCols; c < (half + 1) * kCols; c += 16) {
                float g[16], u[16];
                tmem_ld16(trow + c, g);
                if (GU) tmem_ld16(trow + kN + c, u);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c + j;
                    if (n >= nvalid) break;
                    const int p = p0 + n;
                    if (GU) {
                        a.hout[(size_t)p * a.I + r0 + r] = float_to_bf16_bits(silu(g[j]) * u[j]);
                    } else {
                        a.o[(size_t)p * a.H + r0 + r] = g[j];
                    }
                }
            }
        }
        tc_fence_before_sync();
        __syncthreads();
        if (s_abort) abort = 1;
        cur = ng;
    }
    // no MMA may still write tensor memory when it is freed
    if (tid == 0 && chunk) {
        const int sl = (chunk - 1) & 1;
        int dummy = 0;
        tc_wait(a, &mma_bar[sl], (commits[sl] - 1) & 1, dummy);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Work items per expert: ceil(cnt/kN) token tiles x (rows/kM) row tiles, for
// the gate/up phase (rows = I) and the down phase (rows = H); exclusive scans.
__global__ void tc_plan_kernel(const int32_t *__restrict__ cnt, int E, int I, int H,
                               int32_t *__restrict__ gu_off, int32_t *__restrict__ dn_off)
{
    __shared__ int s_gu[HFQ_MAX_EXPERTS], s_dn[HFQ_MAX_EXPERTS];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int tiles = (cnt[e] + kN - 1) / kN;
        s_gu[e] = tiles * (I / kM);
        s_dn[e] = tiles * (H / kM);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int a = 0, b = 0;
        for (int e = 0; e < E; ++e) {
            gu_off[e] = a; dn_off[e] = b;
            a += s_gu[e]; b += s_dn[e];
        }
        gu_off[E] = a; dn_off[E] = b;
    }
}

// pos[perm[q]] = q (the gate/up kernel reads bf16 x through perm itself).
__global__ void tc_pos_kernel(const int32_t *__restrict__ perm, int P, int32_t *__restrict__ pos)
{
    for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < P; q += gridDim.x * blockDim.x)
        pos[perm[q]] = q;
}

// X_perm[q] = x[token of pair perm[q]] as bf16 (16 bytes per thread step);
// pos[perm[q]] = q.
__global__ void tc_gather_kernel(const void *__restrict__ x, int x_f32, const int32_t *__restrict__ perm,
                                 int P, int k, int H, uint16_t *__restrict__ xp, int32_t *__restrict__ pos)
{
    const size_t n8 = (size_t)P * H / 8;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t q = i / (H / 8), c = (i - q * (H / 8)) * 8;
        if (c == 0) pos[perm[q]] = (int32_t)q;
        const size_t src = (size_t)(perm[q] / k) * H + c;
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
__global__ void tc_combine_kernel(const float *__restrict__ o, const int32_t *__restrict__ pos,
                                  const float *__restrict__ wts, int T, int k, int H, float *__restrict__ y,
                                  uint16_t *__restrict__ yb)
{
    const size_t n4 = (size_t)T * H / 4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t t = i / (H / 4), c = (i - t * (H / 4)) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const float w = wts[t * k + j];
            const float4 v = __ldg(reinterpret_cast<const float4 *>(o + (size_t)pos[t * k + j] * H + c));
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
    }
    return n;
}

}  // namespace

size_t tc_workspace_bytes(int T, int k, int H, int I, int E)
{
    const size_t P = (size_t)T * k;
    auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
    return r256(P * H * 2) + r256(P * I * 2) + 2 * r256((size_t)(E + 1) * 4) + r256(P * H * 4) + r256(P * 4);
}

bool tc_supported(int H, int I)
{
    return H % kM == 0 && I % kM == 0 && H % kKC == 0 && I % kKC == 0;
}

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
    uint16_t *hp = reinterpret_cast<uint16_t *>(w);
    w += r256(P * I * 2);
    int32_t *gu_off = reinterpret_cast<int32_t *>(w);
    w += r256((size_t)(E + 1) * 4);
    int32_t *dn_off = reinterpret_cast<int32_t *>(w);
    w += r256((size_t)(E + 1) * 4);
    float *ob = reinterpret_cast<float *>(w);
    w += r256(P * H * 4);
    int32_t *pos = reinterpret_cast<int32_t *>(w);

    static bool attr = false;
    const int smem_gu = 2 * 3 * kTileBytes, smem_dn = 2 * 2 * kTileBytes;
    if (!attr) {
        cudaFuncSetAttribute(tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_gu);
        cudaFuncSetAttribute(tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dn);
        attr = true;
    }
    tc_plan_kernel<<<1, 512, 0, s>>>(cnt, E, I, H, gu_off, dn_off);
    const size_t n8 = P * H / 8;
    if (x_f32)
        tc_gather_kernel<<<(unsigned)std::min<size_t>((n8 + 255) / 256, (size_t)tc_sms() * 16), 256, 0, s>>>(
            x, 1, perm, (int)P, k, H, xp, pos);
    else
        tc_pos_kernel<<<(unsigned)std::min<size_t>((P + 255) / 256, (size_t)tc_sms() * 4), 256, 0, s>>>(
            perm, (int)P, pos);
    TcArgs a;
    a.eptr = L.expert_ptr; a.cnt = cnt; a.off = off; a.perm = perm; a.wts = wts;
    a.status = status; a.timeout_ns = timeout_ns; a.E = E; a.H = H; a.I = I; a.k = k;
    a.xin = x_f32 ? xp : static_cast<const uint16_t *>(x); a.x_direct = x_f32 ? 0 : 1;
    a.hout = hp; a.o = nullptr; a.item_off = gu_off;
    tc_kernel<true><<<tc_sms(), kTcThr, smem_gu, s>>>(a);
    a.xin = hp; a.x_direct = 0; a.hout = nullptr; a.o = ob; a.item_off = dn_off;
    tc_kernel<false><<<tc_sms(), kTcThr, smem_dn, s>>>(a);
    const size_t n4 = (size_t)T * H / 4;
    tc_combine_kernel<<<(unsigned)std::min<size_t>((n4 + 255) / 256, (size_t)tc_sms() * 16), 256, 0, s>>>(
        ob, pos, wts, T, k, H, y, y_bf16);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "tensor-core path launch: %s", cudaGetErrorString(e));
    return HFQ_OK;
}

}  // namespace hfq
