// topk.cuh - routing of one token by one warp: the k largest router logits
// (ties to the lower expert index) and their softmax over the selected k
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

// Routing of one token by all kWarps warps of a CTA: warp w takes the top k
// of experts [w * E / kWarps, (w + 1) * E / kWarps) into cand_key/cand_e
// (shared, [kWarps][k]); after a block barrier, warp 0 merges the kWarps * k
// candidates.  Candidates of equal keys are in expert order (warp, then
// round), so the merge's lowest-candidate tie rule is the lowest expert, and
// the selection and weights are those of warp_route.  E % (kWarps * 32) == 0
// or E / kWarps <= 32; k <= 16.  Warp 0 lane j < k returns (e_j, w_j).
// kShared: `row` is in shared memory (plain loads instead of the read-only
// global path).
template <int kWarps, bool kShared = false>
__device__ __forceinline__ void cta_route(const float *row, int E, int k, uint32_t *cand_key, int *cand_e,
                                          int &my_e, float &my_w)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = E / kWarps, base = warp * C;
    int e_ = -1;
    float w_ = 0.0f;
    auto keep = [&](int j, int e, uint32_t m) {
        if (lane == 0) {
            cand_key[warp * k + j] = m;
            cand_e[warp * k + j] = e;
        }
    };
    auto key_g = [&](int c) { return order_key(kShared ? row[base + c] : __ldg(row + base + c)); };
    auto id_g = [&](int c) { return base + c; };
    if (C <= 32) warp_topk_core<1>(key_g, id_g, C, k, e_, w_, keep);
    else warp_topk_core<2>(key_g, id_g, C, k, e_, w_, keep);
    __syncthreads();
    if (warp == 0) {
        const int n = kWarps * k;
        auto key_s = [&](int c) { return cand_key[c]; };
        auto id_s = [&](int c) { return cand_e[c]; };
        auto none = [](int, int, uint32_t) {};
        if (n <= 64) warp_topk_core<2>(key_s, id_s, n, k, my_e, my_w, none);
        else warp_topk_core<4>(key_s, id_s, n, k, my_e, my_w, none);
    }
}

}  // namespace hfq

