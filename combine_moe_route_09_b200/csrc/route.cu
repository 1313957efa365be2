// Router top-K gating: one warp per logits row.
//
// "Efficient and portable mixture-of-experts communication", Introduction:
// each token is sent to the K experts with the highest router scores, and the
// expert outputs are added with weights from the router's distribution.
//
// Each lane holds ceil(E/32) logits of the row (expert e = lane + 32*j) in
// registers as ordered 32-bit keys: ordered() maps fp32 to uint32
// monotonically (after -0.0 -> +0.0), so a larger key is a larger logit.
// Round k of K: the warp max of the keys (redux.sync.max), then the lowest
// expert id holding that key (redux.sync.min over each lane's lowest
// candidate) -- ties go to the lower id -- and that key is cleared to 0,
// below every real key.  The softmax over the K selected logits runs on lanes
// 0..K-1.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

__device__ __forceinline__ uint32_t ordered_bits(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float from_ordered(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

template <int NPER>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int S,
                                                         int E, int K, int32_t *__restrict__ topk_idx,
                                                         float *__restrict__ topk_w) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < S; t += warps) {
        const float *row = logits + (size_t)t * E;
        uint32_t key[NPER];
#pragma unroll
        for (int j = 0; j < NPER; ++j) {
            const int e = lane + 32 * j;
            key[j] = e < E ? ordered_bits(__ldg(row + e)) : 0u;
        }
        uint32_t my_key = 0, top = 0;
        int my_e = 0;
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
        if (lane < K) {
            topk_idx[(size_t)t * K + lane] = my_e;
            topk_w[(size_t)t * K + lane] = __fdiv_rn(ex, sum);
        }
    }
}

template <int NPER>
static cudaError_t launch_route(const float *logits, int S, int E, int K, int32_t *idx, float *w,
                                cudaStream_t st, int sms) {
    const int threads = 256;
    int blocks = (S + 7) / 8;
    const int cap_blocks = sms * 8;
    if (blocks > cap_blocks) blocks = cap_blocks;
    if (blocks < 1) blocks = 1;
    static KernelSlots<decltype(&route_topk_kernel<NPER>)> slots;
    int n_sms = 0, per_sm = 0;
    const cudaError_t e = slots.prepare(&route_topk_kernel<NPER>, threads, 0, &n_sms, &per_sm);
    if (e != cudaSuccess) return e;
    return launch_pdl(route_topk_kernel<NPER>, dim3(blocks), dim3(threads), 0, st, logits, S, E, K, idx, w);
}

cudaError_t launch_route_topk(const float *logits, int S, int E, int K, int32_t *idx, float *w,
                              cudaStream_t st, int sms) {
    const int nper = (E + 31) / 32;
    if (nper <= 1) return launch_route<1>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 2) return launch_route<2>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 4) return launch_route<4>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 8) return launch_route<8>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 12) return launch_route<12>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 16) return launch_route<16>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 24) return launch_route<24>(logits, S, E, K, idx, w, st, sms);
    return launch_route<32>(logits, S, E, K, idx, w, st, sms);
}

// Backward through the gating softmax: for the selected experts
// grad_logits[t, e_k] = w_k (gw_k - sum_j w_j gw_j), 0 for the others.  One warp
// per token: the dense row is zeroed, then lanes k < K write their entries
// (ids outside [0, E) are skipped).
__global__ void __launch_bounds__(256) route_backward_kernel(const int32_t *__restrict__ topk_idx,
                                                             const float *__restrict__ topk_w,
                                                             const float *__restrict__ grad_w, int S, int E,
                                                             int K, float *__restrict__ grad_logits) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < S; t += warps) {
        float w = 0.f, gw = 0.f;
        int e = -1;
        if (lane < K) {
            w = __ldg(topk_w + (size_t)t * K + lane);
            gw = __ldg(grad_w + (size_t)t * K + lane);
            e = __ldg(topk_idx + (size_t)t * K + lane);
        }
        float dot = __fmul_rn(w, gw);
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) dot += __shfl_xor_sync(FULL, dot, m);
        float *row = grad_logits + (size_t)t * E;
        for (int j = lane; j < E; j += 32) row[j] = 0.f;
        __syncwarp();
        if (lane < K && e >= 0 && e < E) row[e] = __fmul_rn(w, __fsub_rn(gw, dot));
    }
}

cudaError_t launch_route_backward(const int32_t *topk_idx, const float *topk_w, const float *grad_w, int S,
                                  int E, int K, float *grad_logits, cudaStream_t st, int sms) {
    const int threads = 256;
    int blocks = (S + 7) / 8;
    if (blocks > sms * 8) blocks = sms * 8;
    if (blocks < 1) blocks = 1;
    static KernelSlots<decltype(&route_backward_kernel)> slots;
    int n_sms = 0, per_sm = 0;
    const cudaError_t e = slots.prepare(&route_backward_kernel, threads, 0, &n_sms, &per_sm);
    if (e != cudaSuccess) return e;
    return launch_pdl(route_backward_kernel, dim3(blocks), dim3(threads), 0, st, topk_idx, topk_w, grad_w, S, E,
                      K, grad_logits);
}

}  // namespace moe
