// Shared device helpers of the sm_100a MoE routing kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

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

__device__ __forceinline__ void set_status(int32_t *status, int bit) {
    if (status) atomicOr(status, bit);
}

// Lanes below this one in the warp.
__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace moe
