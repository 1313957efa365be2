// Internal launchers shared by the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Layout tiling: a CTA of LT_WARPS warps takes LT_TILE consecutive (token, k)
// pairs; each warp takes LT_ITEMS consecutive chunks of 32 pairs.
constexpr int LT_WARPS = 16;
constexpr int LT_ITEMS = 4;
constexpr int LT_THREADS = LT_WARPS * 32;
constexpr int LT_TILE = LT_THREADS * LT_ITEMS;
constexpr size_t LT_HEADER = 256;

inline int layout_tiles(long long npairs) {
    long long t = (npairs + LT_TILE - 1) / LT_TILE;
    return t < 1 ? 1 : (int)t;
}

inline size_t layout_workspace_bytes(int S, int E, int K) {
    const size_t hist = (size_t)layout_tiles((long long)S * K) * (size_t)E * 4;
    return LT_HEADER + ((hist + 255) / 256) * 256;
}

// Fused route + layout + dispatch.  Its workspace is the layout's workspace,
// then (256-byte aligned) the arrival marks [RD_MAX_CTAS] u32 and the per-CTA
// histogram rows [RD_MAX_CTAS][E rounded up to 8] u16.
constexpr int RD_MAX_CTAS = 512;
size_t route_dispatch_workspace_bytes(int S, int E, int K);
// Kernels moe_route_dispatch launches for these sizes on the current device (1 fused, else 3 or 4; -1: CUDA error).
int route_dispatch_kernel_count(int S, int H, int E, int K, int dtype, int quant);
cudaError_t launch_route_dispatch(const float *logits, const void *x, int dtype, int S, int H, int E, int K, int R,
                                  int P, int quant, int32_t *topk_idx, float *topk_w, int32_t *counts,
                                  int32_t *offsets, int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src,
                                  void *xd, float *xs, int64_t cap, void *workspace, int32_t *status,
                                  cudaStream_t st, int sms);

cudaError_t launch_route_topk(const float *logits, int S, int E, int K, int32_t *idx, float *w,
                              cudaStream_t st, int sms);

cudaError_t launch_layout(const int32_t *topk_idx, int S, int E, int K, int R, int P,
                          int32_t *counts, int32_t *offsets, int32_t *rank_offsets,
                          int32_t *slot_of, int32_t *row_src, int64_t cap, void *workspace,
                          int32_t *status, cudaStream_t st);

cudaError_t launch_dispatch(const void *x, int dtype, int S, int H, int K, const int32_t *slot_of,
                            int quant, void *xd, float *xs, int64_t cap, int32_t *status,
                            cudaStream_t st);

cudaError_t launch_combine(const void *y, int dtype, int S, int H, int K, int64_t cap,
                           const int32_t *slot_of, const float *topk_w, const void *shared_out,
                           const void *residual, void *out, void *out_no_routed, int32_t *status,
                           cudaStream_t st);

cudaError_t launch_combine_fp8(const uint8_t *yq, const float *ys, int dtype, int S, int H, int K, int64_t cap,
                               const int32_t *slot_of, const float *topk_w, const void *shared_out,
                               const void *residual, void *out, void *out_no_routed, int32_t *status,
                               cudaStream_t st);

cudaError_t launch_combine_backward(const void *g, const void *gn, const void *y, int dtype, int S, int H,
                                    int K, int64_t cap, const int32_t *slot_of, const float *topk_w,
                                    void *grad_y, float *grad_w, void *grad_skip, int32_t *status,
                                    cudaStream_t st);

cudaError_t launch_route_sigmoid_grouped(const float *logits, const float *bias, int S, int E, int K, int n_group,
                                         int topk_group, int normalize, float scale, int32_t *idx, float *w,
                                         cudaStream_t st, int sms);

cudaError_t launch_wait_selftest(int which, unsigned long long limit_ns, int32_t *status, const unsigned *flag,
                                 cudaStream_t st);

// Kernels moe_dispatch_layout launches for these sizes on the current device (1 or 2; -1: CUDA error).
int layout_kernel_count(int S, int E, int K);

cudaError_t launch_route_weights(const float *topk_w, const int32_t *row_src, int64_t pairs, int64_t cap,
                                 float *out, int32_t *status, cudaStream_t st, int sms);

cudaError_t launch_route_backward(const int32_t *topk_idx, const float *topk_w, const float *grad_w, int S,
                                  int E, int K, float *grad_logits, cudaStream_t st, int sms);

}  // namespace moe
