// moe_dispatch_layout_static: the dispatch layout without a caller-supplied
// workspace, for callers that cannot allocate device memory on the path that
// calls it -- for example a host framework or engine plugin that owns every
// byte of device memory up front and forbids allocation while it executes, or
// a latency-critical loop that must not pay for cudaMalloc (which may
// synchronise the device).  Such a caller still passes its own inputs and
// outputs; only the layout's scratch (the arrival ticket and the per-tile
// histograms) moves into a fixed array that lives in this library.
//
// The scratch is a file-scope __device__ array of MOE_STATIC_LAYOUT_SCRATCH_BYTES
// (1 MiB): every GPU that loads this library holds it until the process exits.
// In host code its name is only a host-side stand-in, never a device address,
// so the device address is looked up with cudaGetSymbolAddress -- once per
// device, with that device current, on the first call made on the device.
// That first call should therefore come before any stream capture.
//
// All calls on a device share the one array and it keeps the previous call's
// contents, so each call clears the part that must start at zero (the ticket
// header) with a memset on its stream.  Calls whose kernels may overlap on the
// GPU -- concurrent streams, or several host threads -- race on the array and
// must be serialised by the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "moe_route.h"

namespace {

static __device__ __align__(256) unsigned char g_layout_scratch[MOE_STATIC_LAYOUT_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_layout_scratch on the current device (looked up once).
cudaError_t scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" MOE_API int moe_dispatch_layout_static(const int32_t *topk_idx, int S, int E, int K, int R,
                                                  int token_padding, int32_t *counts, int32_t *offsets,
                                                  int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src,
                                                  int64_t cap, int32_t *status, void *stream) {
    // The same argument checks as moe_dispatch_layout, minus the workspace ones.
    if (S < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > MOE_MAX_TOPK || R < 1 || E % R != 0 ||
        token_padding < 0 || cap < 0 || cap >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)S * K + (int64_t)E * (token_padding > 0 ? token_padding - 1 : 0) >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !rank_offsets) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!topk_idx || !slot_of)) return MOE_ERR_INVALID_ARG;
    if (cap > 0 && !row_src) return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {topk_idx, counts, offsets, rank_offsets, slot_of, row_src, status};
    for (const void *p : ptrs)
        if (p && !aligned4(p)) return MOE_ERR_INVALID_ARG;
    // Sizes whose scratch would not fit in the built-in array are refused.
    if (moe::layout_workspace_bytes(S, E, K) > (size_t)MOE_STATIC_LAYOUT_SCRATCH_BYTES)
        return MOE_ERR_SCRATCH_TOO_SMALL;

    void *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The ticket header must start at zero; the histograms are fully written before use.
    if (cudaMemsetAsync(scratch, 0, moe::LT_HEADER, st) != cudaSuccess) return MOE_ERR_CUDA;
    const cudaError_t e = moe::launch_layout(topk_idx, S, E, K, R, token_padding, counts, offsets,
                                             rank_offsets, slot_of, row_src, cap, scratch, status, st);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
