// Shared device helpers of the sm_100a MoE routing kernels.
#pragma once

#include <atomic>
#include <mutex>

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "moe_route.h"

namespace moe {

constexpr unsigned FULL = 0xffffffffu;

// ---- 16-byte global memory access -----------------------------------------

struct alignas(16) U4 {
    uint32_t x, y, z, w;
};

// Read-only streaming load: the row is used once by this kernel, so skip L1.
__device__ __forceinline__ U4 ld_nc_v4(const void *p) {
    U4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_v4(void *p, const U4 &v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// ---- number formats ---------------------------------------------------------

// bf16 -> fp32 is exact: the bf16 pattern is the top half of the fp32 pattern.
__device__ __forceinline__ float bf16lo(uint32_t pair) { return __uint_as_float(pair << 16); }
__device__ __forceinline__ float bf16hi(uint32_t pair) { return __uint_as_float(pair & 0xffff0000u); }

// Two fp32 -> packed bf16x2 (a in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}

// Two fp32 -> packed e4m3x2 (a in the low byte), round to nearest even,
// saturating to +-448.  The PTX instruction puts its first source in the
// upper byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float a, float b) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

// Programmatic dependent launch.  Every kernel of this library is launched
// with programmatic stream serialisation, so it may start while the kernel
// before it on the stream is still running.  pdl_wait() blocks until that
// kernel (and so everything before it) has completed and its memory is
// visible; no kernel touches its inputs or outputs before it.  pdl_trigger()
// lets the next kernel start launching; kernels call it only after their own
// pdl_wait(), so work two launches back is always complete when a kernel
// starts.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_status(int32_t *status, int bit) {
    if (status) atomicOr(status, bit);
}

// Lanes below this one in the warp.
__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Launches a kernel with programmatic stream serialisation (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// A yes/no launch setting kept per device (up to 64 devices; devices past that
// share the last entry): starts true and is switched off for that device alone
// when the driver refuses the launch form it guards.
struct PerDeviceFlag {
    static constexpr int N = 64;
    std::atomic<int> off[N] = {};
    static int dev_index() {
        int d = 0;
        if (cudaGetDevice(&d) != cudaSuccess || d < 0) d = 0;
        return d < N ? d : N - 1;
    }
    bool on() const { return off[dev_index()].load(std::memory_order_relaxed) == 0; }
    void disable() { off[dev_index()].store(1, std::memory_order_relaxed); }
};

// Launch facts per (device, kernel, block size, dynamic shared memory size):
// how many CTAs fit on one SM.  A kernel's opt-in limit for dynamic shared
// memory is one setting per device and kernel that the last call wins, so it
// is only ever raised, to the largest size requested so far, and every smaller
// launch stays within it.  Up to 32 (device, kernel) pairs and 32 occupancy
// answers are cached; beyond that the calls simply run again.  A mutex guards
// the tables against concurrent host threads.
template <typename Kern>
struct KernelSlots {
    // One object may serve several kernels of the same signature (template
    // instances), so every cached fact is keyed by (device, kernel).
    static constexpr int N = 32;
    struct Attr {
        int dev = -1;
        Kern kern = nullptr;
        size_t limit = 0;  // largest dynamic shared memory set so far (the attribute only grows)
    };
    struct Occ {
        int dev = -1;
        Kern kern = nullptr;
        int threads = 0;
        size_t smem = 0;
        int sms = 0, per_sm = 0;
    };
    Attr attr[N];
    Occ occ[N];
    int n_attr = 0, next_occ = 0;
    std::mutex mu;

    cudaError_t prepare(Kern kern, int threads, size_t bytes, int *n_sms, int *n_per_sm) {
        int d = 0;
        cudaError_t e = cudaGetDevice(&d);
        if (e != cudaSuccess) return e;
        std::lock_guard<std::mutex> lock(mu);
        Attr *a = nullptr;
        for (int i = 0; i < n_attr; ++i)
            if (attr[i].dev == d && attr[i].kern == kern) a = &attr[i];
        if (!a) {
            // First use on this device: ask for the largest shared-memory carveout,
            // so consecutive kernels never wait for an L1/shared split to be
            // reconfigured.
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
            if (n_attr < N) {
                a = &attr[n_attr++];
                a->dev = d;
                a->kern = kern;
            }
        }
        if (!a || bytes > a->limit) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
            if (e != cudaSuccess) return e;
            if (a) a->limit = bytes;
        }
        for (int i = 0; i < N; ++i) {
            const Occ &o = occ[i];
            if (o.dev == d && o.kern == kern && o.threads == threads && o.smem == bytes) {
                *n_sms = o.sms;
                *n_per_sm = o.per_sm;
                return cudaSuccess;
            }
        }
        int s = 0, p = 0;
        e = cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, d);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p, kern, threads, bytes);
        if (e != cudaSuccess) return e;
        if (p < 1) p = 1;
        Occ &o = occ[next_occ++ % N];
        o.dev = d;
        o.kern = kern;
        o.threads = threads;
        o.smem = bytes;
        o.sms = s;
        o.per_sm = p;
        *n_sms = s;
        *n_per_sm = p;
        return cudaSuccess;
    }
};

}  // namespace moe
