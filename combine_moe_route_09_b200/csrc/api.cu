// C-ABI entry points: host-side argument checks, then the launches.  Every
// entry point only enqueues work on the caller's stream.
//
// Each entry point that enqueues GPU work opens an NVTX range named after it
// for the time of the call, so a profiler's timeline labels the launches of
// each step of the path.  NVTX is header-only here: with no tool attached the
// range calls do nothing.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.cuh"
#include "moe_route.h"

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int current_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

int esize(int dtype) { return dtype == MOE_DTYPE_F32 ? 4 : (dtype == MOE_DTYPE_BF16 ? 2 : 0); }

int to_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// NVTX range for the lifetime of one entry-point call.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};

// Activation rows: 16-byte aligned base and a row size that is a multiple of 16 bytes.
bool rows_ok(const void *p, int H, int bytes_per_elem) {
    return p && aligned(p, 16) && ((size_t)H * bytes_per_elem) % 16 == 0;
}

}  // namespace

extern "C" {

const char *moe_error_string(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_CUDA: return "CUDA launch error";
        case MOE_ERR_SCRATCH_TOO_SMALL:
            return "sizes need more scratch than moe_dispatch_layout_static's built-in array";
        default: return "unknown error";
    }
}

int64_t moe_capacity(int S, int E, int K, int token_padding) {
    if (S < 0 || E < 1 || K < 1 || token_padding < 0) return -1;
    return (int64_t)S * K + (int64_t)E * (token_padding > 0 ? token_padding - 1 : 0);
}

int moe_route_topk(const float *logits, int S, int E, int K, int32_t *topk_idx, float *topk_w,
                   void *stream) {
    if (S < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > E || K > MOE_MAX_TOPK)
        return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * E >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_route_topk");
    return to_rc(moe::launch_route_topk(logits, S, E, K, topk_idx, topk_w,
                                        static_cast<cudaStream_t>(stream), current_sms()));
}

int moe_selftest_wait_timeout(int which, unsigned long long limit_ns, int32_t *status, uint32_t *flag,
                              void *stream) {
    if ((which != 0 && which != 1) || limit_ns < 1 || limit_ns > 1000000000ull) return MOE_ERR_INVALID_ARG;
    if (!status || !aligned(status, 4) || (which == 1 && (!flag || !aligned(flag, 4)))) return MOE_ERR_INVALID_ARG;
    const Range range("moe_selftest_wait_timeout");
    return to_rc(moe::launch_wait_selftest(which, limit_ns, status, flag, static_cast<cudaStream_t>(stream)));
}

int moe_dispatch_layout_kernels(int S, int E, int K) {
    if (S < 1 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > MOE_MAX_TOPK || (int64_t)S * K >= ((int64_t)1 << 31)) return 0;
    return moe::layout_kernel_count(S, E, K);
}

int moe_dispatch_route_weights(const float *topk_w, const int32_t *row_src, int S, int K, int64_t cap,
                               float *route_weights, int32_t *status, void *stream) {
    if (S < 0 || K < 1 || K > MOE_MAX_TOPK || cap < 0 || cap >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
    if (cap == 0) return MOE_OK;
    if (!row_src || !route_weights || (S > 0 && !topk_w)) return MOE_ERR_INVALID_ARG;
    if (!aligned(row_src, 4) || !aligned(route_weights, 4) || (topk_w && !aligned(topk_w, 4)) ||
        (status && !aligned(status, 4)))
        return MOE_ERR_INVALID_ARG;
    const Range range("moe_dispatch_route_weights");
    return to_rc(moe::launch_route_weights(topk_w, row_src, (int64_t)S * K, cap, route_weights, status,
                                           static_cast<cudaStream_t>(stream), current_sms()));
}

int moe_route_sigmoid_grouped(const float *logits, const float *bias, int S, int E, int K, int n_group,
                              int topk_group, int normalize, float scale, int32_t *topk_idx, float *topk_w,
                              void *stream) {
    if (S < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > E || K > MOE_MAX_TOPK) return MOE_ERR_INVALID_ARG;
    if (n_group < 1 || n_group > MOE_MAX_GROUPS || E % n_group != 0) return MOE_ERR_INVALID_ARG;
    if (n_group > 1 && (E / n_group < 2 || topk_group < 1 || topk_group > n_group ||
                        (int64_t)topk_group * (E / n_group) < K))
        return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) || (bias && !aligned(bias, 4)))
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * E >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_route_sigmoid_grouped");
    return to_rc(moe::launch_route_sigmoid_grouped(logits, bias, S, E, K, n_group, n_group > 1 ? topk_group : 1,
                                                   normalize, scale, topk_idx, topk_w,
                                                   static_cast<cudaStream_t>(stream), current_sms()));
}

size_t moe_dispatch_layout_workspace(int S, int E, int K) {
    if (S < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > MOE_MAX_TOPK) return 0;
    if ((int64_t)S * K >= ((int64_t)1 << 31)) return 0;
    return moe::layout_workspace_bytes(S, E, K);
}

int moe_dispatch_layout(const int32_t *topk_idx, int S, int E, int K, int R, int token_padding,
                        int32_t *counts, int32_t *offsets, int32_t *rank_offsets, int32_t *slot_of,
                        int32_t *row_src, int64_t cap, void *workspace, size_t workspace_bytes,
                        int32_t *status, void *stream) {
    if (S < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > MOE_MAX_TOPK || R < 1 || E % R != 0 ||
        token_padding < 0 || cap < 0 || cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    // The padded layout must be addressable with int32 rows whatever the routing.
    if ((int64_t)S * K + (int64_t)E * (token_padding > 0 ? token_padding - 1 : 0) >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !rank_offsets || !workspace) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!topk_idx || !slot_of)) return MOE_ERR_INVALID_ARG;
    if (cap > 0 && !row_src) return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || workspace_bytes < moe::layout_workspace_bytes(S, E, K))
        return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {topk_idx, counts, offsets, rank_offsets, slot_of, row_src, status};
    for (const void *p : ptrs)
        if (p && !aligned(p, 4)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_dispatch_layout");
    return to_rc(moe::launch_layout(topk_idx, S, E, K, R, token_padding, counts, offsets,
                                    rank_offsets, slot_of, row_src, cap, workspace, status,
                                    static_cast<cudaStream_t>(stream)));
}

size_t moe_route_dispatch_workspace(int S, int E, int K) {
    if (S < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > MOE_MAX_TOPK) return 0;
    if ((int64_t)S * K >= ((int64_t)1 << 31)) return 0;
    return moe::route_dispatch_workspace_bytes(S, E, K);
}

int moe_route_dispatch_kernels(int S, int H, int E, int K, int dtype, int quant) {
    if (S < 1 || H < 1 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > E || K > MOE_MAX_TOPK || esize(dtype) == 0 ||
        (quant != MOE_QUANT_NONE && quant != MOE_QUANT_FP8_E4M3_B128) || (int64_t)S * K >= ((int64_t)1 << 31))
        return 0;
    return moe::route_dispatch_kernel_count(S, H, E, K, dtype, quant);
}

int moe_route_dispatch(const float *logits, const void *x, int dtype, int S, int H, int E, int K, int R,
                       int token_padding, int quant, int32_t *topk_idx, float *topk_w, int32_t *counts,
                       int32_t *offsets, int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src, void *xd,
                       float *xs, int64_t cap, void *workspace, size_t workspace_bytes, int32_t *status,
                       void *stream) {
    // the checks of moe_route_topk, moe_dispatch_layout and moe_dispatch together
    const int b = esize(dtype);
    if (S < 0 || H < 1 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > E || K > MOE_MAX_TOPK || R < 1 ||
        E % R != 0 || token_padding < 0 || b == 0 || cap < 0 || cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (quant != MOE_QUANT_NONE && quant != MOE_QUANT_FP8_E4M3_B128) return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * K + (int64_t)E * (token_padding > 0 ? token_padding - 1 : 0) >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * E >= ((int64_t)1 << 40) || (int64_t)S * H >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !rank_offsets || !workspace) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!logits || !topk_idx || !topk_w || !slot_of || !rows_ok(x, H, b))) return MOE_ERR_INVALID_ARG;
    if (cap > 0 && !row_src) return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || workspace_bytes < moe::route_dispatch_workspace_bytes(S, E, K))
        return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {logits, topk_idx, topk_w, counts, offsets, rank_offsets, slot_of, row_src, status};
    for (const void *p : ptrs)
        if (p && !aligned(p, 4)) return MOE_ERR_INVALID_ARG;
    if (quant == MOE_QUANT_NONE) {
        if (xs || (cap > 0 && S > 0 && !rows_ok(xd, H, b))) return MOE_ERR_INVALID_ARG;
    } else {
        if (H % 128 != 0 || (cap > 0 && S > 0 && (!rows_ok(xd, H, 1) || !xs || !aligned(xs, 4))))
            return MOE_ERR_INVALID_ARG;
    }
    const Range range("moe_route_dispatch");
    return to_rc(moe::launch_route_dispatch(logits, x, dtype, S, H, E, K, R, token_padding, quant, topk_idx, topk_w,
                                            counts, offsets, rank_offsets, slot_of, row_src, xd, xs, cap, workspace,
                                            status, static_cast<cudaStream_t>(stream), current_sms()));
}

int moe_dispatch(const void *x, int dtype, int S, int H, int K, const int32_t *slot_of, int quant,
                 void *xd, float *xs, int64_t cap, int32_t *status, void *stream) {
    const int b = esize(dtype);
    if (S < 0 || H < 1 || K < 1 || K > MOE_MAX_TOPK || b == 0 || cap < 0 || cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (quant != MOE_QUANT_NONE && quant != MOE_QUANT_FP8_E4M3_B128) return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!slot_of || !aligned(slot_of, 4) || (status && !aligned(status, 4))) return MOE_ERR_INVALID_ARG;
    if (!rows_ok(x, H, b)) return MOE_ERR_INVALID_ARG;
    if (quant == MOE_QUANT_NONE) {
        if (xs || (cap > 0 && !rows_ok(xd, H, b))) return MOE_ERR_INVALID_ARG;
    } else {
        if (H % 128 != 0 || (cap > 0 && (!rows_ok(xd, H, 1) || !xs || !aligned(xs, 4))))
            return MOE_ERR_INVALID_ARG;
    }
    if ((int64_t)S * H >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_dispatch");
    return to_rc(moe::launch_dispatch(x, dtype, S, H, K, slot_of, quant, xd, xs, cap, status,
                                      static_cast<cudaStream_t>(stream)));
}

int moe_combine_dual_residual(const void *y, int dtype, int S, int H, int K, int64_t cap,
                              const int32_t *slot_of, const float *topk_w, const void *shared_out,
                              const void *residual, void *residual_out,
                              void *residual_no_routed_out, int32_t *status, void *stream) {
    const int b = esize(dtype);
    if (S < 0 || H < 1 || K < 1 || K > MOE_MAX_TOPK || b == 0 || cap < 0 || cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (residual_no_routed_out && !(shared_out && residual)) return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!slot_of || !topk_w || !aligned(slot_of, 4) || !aligned(topk_w, 4)) return MOE_ERR_INVALID_ARG;
    if (status && !aligned(status, 4)) return MOE_ERR_INVALID_ARG;
    if ((cap > 0 && !rows_ok(y, H, b)) || !rows_ok(residual_out, H, b)) return MOE_ERR_INVALID_ARG;
    if (shared_out && !rows_ok(shared_out, H, b)) return MOE_ERR_INVALID_ARG;
    if (residual && !rows_ok(residual, H, b)) return MOE_ERR_INVALID_ARG;
    if (residual_no_routed_out && !rows_ok(residual_no_routed_out, H, b)) return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * H >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_combine_dual_residual");
    return to_rc(moe::launch_combine(y, dtype, S, H, K, cap, slot_of, topk_w, shared_out, residual,
                                     residual_out, residual_no_routed_out, status,
                                     static_cast<cudaStream_t>(stream)));
}

int moe_combine_fp8_dual_residual(const uint8_t *yq, const float *ys, int dtype, int S, int H, int K, int64_t cap,
                                  const int32_t *slot_of, const float *topk_w, const void *shared_out,
                                  const void *residual, void *residual_out, void *residual_no_routed_out,
                                  int32_t *status, void *stream) {
    const int b = esize(dtype);
    if (S < 0 || H < 1 || H % 512 != 0 || K < 1 || K > MOE_MAX_TOPK || b == 0 || cap < 0 ||
        cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (residual_no_routed_out && !(shared_out && residual)) return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!slot_of || !topk_w || !aligned(slot_of, 4) || !aligned(topk_w, 4)) return MOE_ERR_INVALID_ARG;
    if (status && !aligned(status, 4)) return MOE_ERR_INVALID_ARG;
    if (cap > 0 && (!rows_ok(yq, H, 1) || !ys || !aligned(ys, 16))) return MOE_ERR_INVALID_ARG;
    if (!rows_ok(residual_out, H, b)) return MOE_ERR_INVALID_ARG;
    if (shared_out && !rows_ok(shared_out, H, b)) return MOE_ERR_INVALID_ARG;
    if (residual && !rows_ok(residual, H, b)) return MOE_ERR_INVALID_ARG;
    if (residual_no_routed_out && !rows_ok(residual_no_routed_out, H, b)) return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * H >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_combine_fp8_dual_residual");
    return to_rc(moe::launch_combine_fp8(yq, ys, dtype, S, H, K, cap, slot_of, topk_w, shared_out, residual,
                                         residual_out, residual_no_routed_out, status,
                                         static_cast<cudaStream_t>(stream)));
}

int moe_combine_dual_residual_backward(const void *grad_out, const void *grad_no_routed, const void *y,
                                       int dtype, int S, int H, int K, int64_t cap, const int32_t *slot_of,
                                       const float *topk_w, void *grad_y, float *grad_w, void *grad_skip,
                                       int32_t *status, void *stream) {
    const int b = esize(dtype);
    if (S < 0 || H < 1 || K < 1 || K > MOE_MAX_TOPK || b == 0 || cap < 0 || cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!slot_of || !topk_w || !grad_w || !aligned(slot_of, 4) || !aligned(topk_w, 4) || !aligned(grad_w, 4))
        return MOE_ERR_INVALID_ARG;
    if (status && !aligned(status, 4)) return MOE_ERR_INVALID_ARG;
    if (!rows_ok(grad_out, H, b)) return MOE_ERR_INVALID_ARG;
    if (cap > 0 && (!rows_ok(y, H, b) || !rows_ok(grad_y, H, b))) return MOE_ERR_INVALID_ARG;
    if (grad_no_routed && !rows_ok(grad_no_routed, H, b)) return MOE_ERR_INVALID_ARG;
    if (grad_skip && !rows_ok(grad_skip, H, b)) return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * H >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_combine_dual_residual_backward");
    return to_rc(moe::launch_combine_backward(grad_out, grad_no_routed, y, dtype, S, H, K, cap, slot_of, topk_w,
                                              grad_y, grad_w, grad_skip, status, static_cast<cudaStream_t>(stream)));
}

int moe_dispatch_backward(const void *grad_xd, int dtype, int S, int H, int K, int64_t cap,
                          const int32_t *slot_of, void *grad_x, int32_t *status, void *stream) {
    const int b = esize(dtype);
    if (S < 0 || H < 1 || K < 1 || K > MOE_MAX_TOPK || b == 0 || cap < 0 || cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!slot_of || !aligned(slot_of, 4) || (status && !aligned(status, 4))) return MOE_ERR_INVALID_ARG;
    if ((cap > 0 && !rows_ok(grad_xd, H, b)) || !rows_ok(grad_x, H, b)) return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * H >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    // the combine with unit weights and no epilogue: grad_x[t] = sum_k grad_xd[slot]
    const Range range("moe_dispatch_backward");
    return to_rc(moe::launch_combine(grad_xd, dtype, S, H, K, cap, slot_of, nullptr, nullptr, nullptr, grad_x,
                                     nullptr, status, static_cast<cudaStream_t>(stream)));
}

int moe_route_topk_backward(const int32_t *topk_idx, const float *topk_w, const float *grad_w, int S, int E,
                            int K, float *grad_logits, void *stream) {
    if (S < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > E || K > MOE_MAX_TOPK) return MOE_ERR_INVALID_ARG;
    if (S == 0) return MOE_OK;
    if (!topk_idx || !topk_w || !grad_w || !grad_logits) return MOE_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4) || !aligned(grad_w, 4) || !aligned(grad_logits, 4))
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * E >= ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
    const Range range("moe_route_topk_backward");
    return to_rc(moe::launch_route_backward(topk_idx, topk_w, grad_w, S, E, K, grad_logits,
                                            static_cast<cudaStream_t>(stream), current_sms()));
}

}  // extern "C"
