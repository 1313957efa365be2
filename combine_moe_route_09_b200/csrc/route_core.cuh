// Router top-K over one logits row, done by one warp: shared by the router
// kernel (route.cu) and the fused route + dispatch kernel, so both produce the
// same experts and the same weights bit for bit.
//
// Each lane holds ceil(E/32) logits of the row (expert e = lane + 32*j) in
// registers as ordered 32-bit keys: ordered_bits() maps fp32 to uint32
// monotonically (after -0.0 -> +0.0), so a larger key is a larger logit.
// Round k of K: the warp max of the keys (redux.sync.max), then the lowest
// expert id holding that key (redux.sync.min over each lane's lowest
// candidate) -- ties go to the lower id -- and that key is cleared to 0,
// below every real key.  The softmax over the K selected logits runs on lanes
// 0..K-1: w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0).
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ uint32_t ordered_bits(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float from_ordered(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// The row's logits as ordered keys; experts past E get key 0.
template <int NPER>
__device__ __forceinline__ void load_route_keys(const float *__restrict__ row, int E, int lane, uint32_t (&key)[NPER]) {
#pragma unroll
    for (int j = 0; j < NPER; ++j) {
        const int e = lane + 32 * j;
        key[j] = e < E ? ordered_bits(__ldg(row + e)) : 0u;
    }
}

// K rounds of max / lowest id; lane k < K gets the k-th expert and its weight.
template <int NPER>
__device__ __forceinline__ void topk_softmax(uint32_t (&key)[NPER], int K, int lane, int &my_e, float &my_w) {
    uint32_t my_key = 0, top = 0;
    my_e = 0;
    for (int k = 0; k < K; ++k) {
        uint32_t m = key[0];
#pragma unroll
        for (int j = 1; j < NPER; ++j) m = max(m, key[j]);
        const uint32_t best = __reduce_max_sync(FULL, m);
        uint32_t cand = 0xffffffffu;
#pragma unroll
        for (int j = NPER - 1; j >= 0; --j) cand = key[j] == best ? (uint32_t)(lane + 32 * j) : cand;
        const uint32_t win = __reduce_min_sync(FULL, cand);
        if (k == 0) top = best;
        if (lane == k) {
            my_key = best;
            my_e = (int)win;
        }
#pragma unroll
        for (int j = 0; j < NPER; ++j) key[j] = (uint32_t)(lane + 32 * j) == win ? 0u : key[j];
    }
    const float ex = lane < K ? expf(from_ordered(my_key) - from_ordered(top)) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
    my_w = __fdiv_rn(ex, sum);
}

}  // namespace moe
