// topk.cuh - routing of one token, by one warp or by a whole CTA: the k
// largest router logits (ties to the lower expert index) and their softmax
// over the selected k
// (hipfire offload explainer, opening section: top-k experts per token,
// weights renormalised over the chosen ones).
#pragma once

#include <cstdint>

namespace hfq {

// Order-preserving map float -> uint32 (larger float, larger key; -0 as +0).
// Key 0 lies below every real key.
__device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Lane i holds candidates i*M .. i*M+M-1 of n (keys from `key_of(c)`,
// order_key values; ids from `id_of(c)`, ascending with c among equal keys)
// and keeps its three largest untaken keys in registers (k0 >= k1 >= k2;
// equal keys in candidate order).  Each of the k rounds takes the warp max
// of the lanes' k0, the lowest lane winning ties (the lowest candidate); the
// winner shifts its cache (selects, no branch) and, once three of its keys
// are taken, rescans its M keys on a warp-uniform branch.
// `on_round(j, id, key)` runs on the whole warp right after round j has
// selected candidate `id`.  Lane j < k returns the j-th selected id and its
// weight exp(v_j - v_0) / sum_i<k exp(v_i - v_0); other lanes return -1.
template <int M, class Key, class Id, class F>
__device__ __forceinline__ void warp_topk_core(Key &&key_of, Id &&id_of, int n, int k, int &my_e, float &my_w,
                                               F &&on_round)
{
    const int lane = threadIdx.x & 31;
    uint32_t key[M];
#pragma unroll
    for (int i = 0; i < M; ++i) {
        const int c = lane * M + i;
        key[i] = c < n ? key_of(c) : 0u;
    }
    uint32_t k0, k1, k2;
    int i0, i1, i2;
    auto top3 = [&](uint32_t taken) {
        k0 = k1 = k2 = 0u;
        i0 = i1 = i2 = 0;
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const uint32_t x = (taken >> i & 1u) ? 0u : key[i];
            const bool g0 = x > k0, g1 = x > k1, g2 = x > k2;
            k2 = g1 ? k1 : (g2 ? x : k2);
            i2 = g1 ? i1 : (g2 ? i : i2);
            k1 = g0 ? k0 : (g1 ? x : k1);
            i1 = g0 ? i0 : (g1 ? i : i1);
            k0 = g0 ? x : k0;
            i0 = g0 ? i : i0;
        }
    };
    top3(0u);
    uint32_t taken = 0u;
    int wins = 0;
    float v0 = 0.0f, s = 0.0f, my_ex = 0.0f;
    my_e = -1;
    for (int j = 0; j < k; ++j) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, k0);
        const unsigned ball = __ballot_sync(0xffffffffu, k0 == m);
        const int win = __ffs(ball) - 1;
        const int c = lane * M + i0;
        const int e = __shfl_sync(0xffffffffu, c < n ? id_of(c) : -1, win);
        const bool won = lane == win;
        taken |= won ? 1u << i0 : 0u;
        k0 = won ? k1 : k0;
        i0 = won ? i1 : i0;
        k1 = won ? k2 : k1;
        i1 = won ? i2 : i1;
        k2 = won ? 0u : k2;
        wins += won ? 1 : 0;
        if (M > 3 && __any_sync(0xffffffffu, won && wins == 3)) {
            if (won) {
                top3(taken);
                wins = 0;
            }
        }
        const float v = key_value(m);
        if (j == 0) v0 = v;
        const float ex = __expf(v - v0);
        s += ex;
        if (lane == j) { my_ex = ex; my_e = e; }
        on_round(j, e, m);
    }
    my_w = my_ex / s;
}

// The k largest of E logits `row`, lane i holding experts i*M .. i*M+M-1.
template <int M, class F>
__device__ __forceinline__ void warp_topk_rounds(const float *__restrict__ row, int E, int k, int &my_e,
                                                 float &my_w, F &&on_round)
{
    warp_topk_core<M>([&](int c) { return order_key(__ldg(row + c)); }, [](int c) { return c; }, E, k, my_e,
                      my_w, [&](int j, int e, uint32_t) { on_round(j, e); });
}

// warp_topk_rounds with M chosen from E (E <= 512).
template <class F>
__device__ __forceinline__ void warp_route_rounds(const float *row, int E, int k, int &my_e, float &my_w,
                                                  F &&on_round)
{
    if (E <= 32) warp_topk_rounds<1>(row, E, k, my_e, my_w, on_round);
    else if (E <= 64) warp_topk_rounds<2>(row, E, k, my_e, my_w, on_round);
    else if (E <= 128) warp_topk_rounds<4>(row, E, k, my_e, my_w, on_round);
    else if (E <= 256) warp_topk_rounds<8>(row, E, k, my_e, my_w, on_round);
    else warp_topk_rounds<16>(row, E, k, my_e, my_w, on_round);
}

__device__ __forceinline__ void warp_route(const float *row, int E, int k, int &my_e, float &my_w)
{
    warp_route_rounds(row, E, k, my_e, my_w, [](int, int) {});
}

// Routing of one token by a whole CTA of kThreads threads by ranks (E <=
// 2 kThreads, k <= 16): every logit gets the 64-bit key
// (order_key(v) << 32) | (0xFFFFFFFF - e), unique and larger for the better
// expert (equal logits: the lower index first), and an expert's rank is the
// number of larger keys.  Step 1 ranks each expert within its group of 64
// (keys in shared memory, read by broadcast, 0 past E); the k best of each
// group are the candidates.  Step 2 ranks the candidates among themselves:
// the k best candidates are the k best experts, the one of rank r taking
// slot r.  The selection and the weights are those of warp_route: warp 0
// lane j < k returns e_j and w_j = exp(v_j - v_0) / s, s = sum over i < k of
// exp(v_i - v_0) added in slot order; other threads return -1.
// keys: shared [E rounded up to 64], cand: shared [ceil(E / 64) * k rounded
// up to 8], sel: shared [k]; keys and cand 16-byte aligned.
template <int kThreads, class LogitOf>
__device__ __forceinline__ void cta_route_rank(LogitOf &&logit_of, int E, int k, uint64_t *keys, uint64_t *cand,
                                               uint64_t *sel, int &my_e, float &my_w)
{
    const int tid = threadIdx.x;
    const int E64 = (E + 63) & ~63, nc = ((E + 63) >> 6) * k, nc8 = (nc + 7) & ~7;
    for (int e = tid; e < E64; e += kThreads)
        keys[e] = e < E ? ((uint64_t)order_key(logit_of(e)) << 32) | (0xFFFFFFFFu - (uint32_t)e) : 0ull;
    for (int c = tid; c < nc8; c += kThreads) cand[c] = 0ull;      // below every key
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {
        const uint64_t K = keys[e];
        const ulonglong2 *g = reinterpret_cast<const ulonglong2 *>(keys + (e & ~63));
        int r = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const ulonglong2 p = g[j];
            r += (p.x > K ? 1 : 0) + (p.y > K ? 1 : 0);
        }
        if (r < k) cand[(e >> 6) * k + r] = K;
    }
    __syncthreads();
    for (int c = tid; c < nc; c += kThreads) {
        const uint64_t K = cand[c];
        const ulonglong2 *g = reinterpret_cast<const ulonglong2 *>(cand);
        int r = 0;
#pragma unroll 4
        for (int j = 0; j < nc8 / 2; ++j) {
            const ulonglong2 p = g[j];
            r += (p.x > K ? 1 : 0) + (p.y > K ? 1 : 0);
        }
        if (K != 0ull && r < k) sel[r] = K;
    }
    __syncthreads();
    my_e = -1;
    my_w = 0.0f;
    if (tid < 32) {
        const float v0 = key_value((uint32_t)(sel[0] >> 32));
        float s = 0.0f, mine = 0.0f;
        for (int j = 0; j < k; ++j) {
            const float ex = __expf(key_value((uint32_t)(sel[j] >> 32)) - v0);
            s += ex;
            mine = j == tid ? ex : mine;
        }
        if (tid < k) {
            my_e = (int)(0xFFFFFFFFu - (uint32_t)sel[tid]);
            my_w = mine / s;
        }
    }
}

// Routing of one token by a whole CTA for k <= kThreads / 32 (E <= 2
// kThreads): the same selection and weights as cta_route_rank with far less
// work.  tau = the smallest of the warps' maxima is a lower bound of the
// k-th largest logit (the kThreads / 32 warp maxima are that many distinct
// experts), so only experts with key >= tau can be selected; they are
// gathered (any order) and ranked among themselves by their unique 64-bit
// keys.  surv: shared [E] keys; wmax: shared [kThreads / 32]; n_surv: a
// shared counter; sel: shared [k].  Warp 0 lane j < k returns (e_j, w_j).
template <int kThreads, class LogitOf>
__device__ __forceinline__ void cta_route_small_k(LogitOf &&logit_of, int E, int k, uint64_t *surv, uint32_t *wmax,
                                                  int *n_surv, uint64_t *sel, int &my_e, float &my_w)
{
    constexpr int kWarps = kThreads / 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t key[2];
    uint32_t m = 0u;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int e = tid + i * kThreads;
        key[i] = e < E ? order_key(logit_of(e)) : 0u;
        m = key[i] > m ? key[i] : m;
    }
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == 0) wmax[warp] = m;
    if (tid == 0) *n_surv = 0;
    __syncthreads();
    uint32_t tau = wmax[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) tau = wmax[w] < tau ? wmax[w] : tau;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int e = tid + i * kThreads;
        if (e < E && key[i] >= tau) surv[atomicAdd(n_surv, 1)] = ((uint64_t)key[i] << 32) | (0xFFFFFFFFu - (uint32_t)e);
    }
    __syncthreads();
    const int n = *n_surv;
    for (int c = tid; c < n; c += kThreads) {
        const uint64_t K = surv[c];
        int r = 0;
#pragma unroll 4
        for (int j = 0; j < n; ++j) r += surv[j] > K ? 1 : 0;
        if (r < k) sel[r] = K;
    }
    __syncthreads();
    my_e = -1;
    my_w = 0.0f;
    if (warp == 0) {
        const uint64_t K = lane < k ? sel[lane] : 0ull;
        const float v = key_value((uint32_t)(K >> 32));
        const float v0 = __shfl_sync(0xffffffffu, v, 0);
        const float ex = __expf(v - v0);
        float s = 0.0f;
        for (int j = 0; j < k; ++j) s += __shfl_sync(0xffffffffu, ex, j);
        if (lane < k) {
            my_e = (int)(0xFFFFFFFFu - (uint32_t)K);
            my_w = ex / s;
        }
    }
}

}  // namespace hfq

