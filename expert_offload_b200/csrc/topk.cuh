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

// Lane i holds experts i*M .. i*M+M-1 of `row` (E logits); k rounds of a warp
// max over the lanes' best keys, the lowest lane winning ties, which is the
// lowest expert index.  Lane j < k returns the j-th selected expert and its
// weight exp(v_j - v_0) / sum_i<k exp(v_i - v_0); other lanes return e = -1.
template <int M>
__device__ void warp_topk_lane(const float *__restrict__ row, int E, int k, int &my_e, float &my_w)
{
    const int lane = threadIdx.x & 31;
    uint32_t key[M];
#pragma unroll
    for (int i = 0; i < M; ++i) {
        const int e = lane * M + i;
        key[i] = e < E ? order_key(__ldg(row + e)) : 0u;
    }
    uint32_t taken = 0, bk = key[0];
    int bi = 0;
#pragma unroll
    for (int i = 1; i < M; ++i)
        if (key[i] > bk) { bk = key[i]; bi = i; }
    float v0 = 0.0f, s = 0.0f, my_ex = 0.0f;
    my_e = -1;
    for (int j = 0; j < k; ++j) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
        const unsigned ball = __ballot_sync(0xffffffffu, bk == m);
        const int win = __ffs(ball) - 1;
        const int e = __shfl_sync(0xffffffffu, lane * M + bi, win);
        const float v = key_value(m);
        if (j == 0) v0 = v;
        const float ex = __expf(v - v0);
        s += ex;
        if (lane == j) { my_ex = ex; my_e = e; }
        if (lane == win) {
            taken |= 1u << bi;
            bool any = false;
            bk = 0u; bi = 0;
#pragma unroll
            for (int i = 0; i < M; ++i)
                if (!(taken >> i & 1u) && (!any || key[i] > bk)) { bk = key[i]; bi = i; any = true; }
        }
    }
    my_w = my_ex / s;
}

// warp_topk_lane with M chosen from E (E <= 512).
__device__ __forceinline__ void warp_route(const float *row, int E, int k, int &my_e, float &my_w)
{
    if (E <= 32) warp_topk_lane<1>(row, E, k, my_e, my_w);
    else if (E <= 64) warp_topk_lane<2>(row, E, k, my_e, my_w);
    else if (E <= 128) warp_topk_lane<4>(row, E, k, my_e, my_w);
    else if (E <= 256) warp_topk_lane<8>(row, E, k, my_e, my_w);
    else warp_topk_lane<16>(row, E, k, my_e, my_w);
}

}  // namespace hfq
