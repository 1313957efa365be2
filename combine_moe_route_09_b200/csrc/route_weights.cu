// Routing weights in dispatched order.
//
// MoonEP developer guide, core API example: the dispatch hands each expert its
// rows together with their routing weights, in the same (expert-contiguous)
// order, and the combine consumes them.  Row r of that order came from pair
// row_src[r] = t*K + k of the layout, so its weight is topk_w[t*K + k]; rows
// that no pair fills (padding, unused capacity) get 0.  One thread per row: a
// coalesced read of row_src, a gather from topk_w (S*K*4 bytes, L2-resident),
// a coalesced store.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

__global__ void __launch_bounds__(256)
    route_weights_kernel(const float *__restrict__ topk_w, const int32_t *__restrict__ row_src, int64_t pairs,
                         int64_t cap, float *__restrict__ out, int32_t *status) {
    pdl_wait();
    pdl_trigger();
    bool bad = false;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < cap; r += stride) {
        const int32_t src = __ldg(row_src + r);
        float v = 0.f;
        if (src >= 0) {
            if (src < pairs) v = __ldg(topk_w + src);
            else bad = true;
        }
        out[r] = v;
    }
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0) set_status(status, MOE_STATUS_BAD_SLOT);
}

cudaError_t launch_route_weights(const float *topk_w, const int32_t *row_src, int64_t pairs, int64_t cap,
                                 float *out, int32_t *status, cudaStream_t st, int sms) {
    const int threads = 256;
    int64_t blocks = (cap + threads - 1) / threads;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    if (blocks < 1) blocks = 1;
    return launch_pdl(route_weights_kernel, dim3((unsigned)blocks), dim3(threads), 0, st, topk_w, row_src, pairs,
                      cap, out, status);
}

}  // namespace moe
