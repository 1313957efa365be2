// Dispatch: scatter each token row into the K rows its (token, k) pairs were
// given, optionally quantised to FP8 e4m3 with one fp32 scale per 128 channels.
//
// "Efficient and portable mixture-of-experts communication", Dispatch: tokens
// and their block scaling factors are packed and laid out contiguously per
// expert for the grouped GEMM.  "DeepSeek AI releases DeepEP", Technical
// overview: the dispatch may carry FP8.
//
// One warp per token: the warp reads the row once (16-byte loads, L1 bypassed)
// and writes it K times (16-byte stores), so HBM sees S*H*b bytes read and
// S*K*H*b_out written.  For FP8 a lane owns 16 consecutive channels, so the 8
// lanes of an aligned lane group own one 128-channel block and reduce its amax
// with three xor-shuffles; scale and quotient are IEEE fp32 divisions, the
// conversion is cvt.rn.satfinite.e4m3x2.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int DP_THREADS = 256;
constexpr int DP_WARPS = DP_THREADS / 32;

// Loads the token's K slots into the warp's shared-memory row; bad slots -> -1.
__device__ __forceinline__ void load_slots(int *s_slot, const int32_t *slot_of, int t, int K,
                                           int64_t cap, int lane, int32_t *status) {
    if (lane < K) {
        int s = __ldg(slot_of + (size_t)t * K + lane);
        if ((int64_t)s >= cap) {
            set_status(status, MOE_STATUS_BAD_SLOT);
            s = -1;
        }
        s_slot[lane] = s;
    }
    __syncwarp();
}

// Bit copy of rows of `nunits` 16-byte units (bf16 or fp32 without quantisation).
template <int UNROLL>
__global__ void __launch_bounds__(DP_THREADS)
    dispatch_copy_kernel(const uint8_t *__restrict__ x, int S, int nunits, int K,
                         const int32_t *__restrict__ slot_of, uint8_t *__restrict__ xd, int64_t cap,
                         int32_t *status) {
    __shared__ int s_slot[DP_WARPS][32];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int t = blockIdx.x * DP_WARPS + wl;
    if (t >= S) return;
    load_slots(s_slot[wl], slot_of, t, K, cap, lane, status);
    const size_t row_bytes = (size_t)nunits * 16;
    const uint8_t *src = x + (size_t)t * row_bytes;
    for (int u0 = 0; u0 < nunits; u0 += 32 * UNROLL) {
        U4 v[UNROLL];
#pragma unroll
        for (int j = 0; j < UNROLL; ++j) {
            const int u = u0 + 32 * j + lane;
            if (u < nunits) v[j] = ld_nc_v4(src + (size_t)u * 16);
        }
        for (int k = 0; k < K; ++k) {
            const int s = s_slot[wl][k];
            if (s < 0) continue;
            uint8_t *dst = xd + (size_t)s * row_bytes;
#pragma unroll
            for (int j = 0; j < UNROLL; ++j) {
                const int u = u0 + 32 * j + lane;
                if (u < nunits) st_v4(dst + (size_t)u * 16, v[j]);
            }
        }
    }
}

// 16 channels of one lane -> four e4m3x4 words, given the block scale.
__device__ __forceinline__ U4 quant16(const float (&f)[16], float s) {
    uint32_t w[4];
    if (s == 0.f) {
        // amax == 0: every element is a signed zero; keep the sign.
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t r = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) r |= ((__float_as_uint(f[4 * i + b]) >> 31) << 7) << (8 * b);
            w[i] = r;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = pack_e4m3x2(__fdiv_rn(f[4 * i + 0], s), __fdiv_rn(f[4 * i + 1], s));
            const uint32_t hi = pack_e4m3x2(__fdiv_rn(f[4 * i + 2], s), __fdiv_rn(f[4 * i + 3], s));
            w[i] = lo | (hi << 16);
        }
    }
    return U4{w[0], w[1], w[2], w[3]};
}

// FP8 dispatch.  IN_F32: input rows are fp32 (else bf16).  A lane unit is 16
// channels; nunits = H / 16 is a multiple of 8, so lane groups stay whole.
template <bool IN_F32, int UNROLL>
__global__ void __launch_bounds__(DP_THREADS)
    dispatch_fp8_kernel(const void *__restrict__ x, int S, int H, int K,
                        const int32_t *__restrict__ slot_of, uint8_t *__restrict__ xd,
                        float *__restrict__ xs, int64_t cap, int32_t *status) {
    __shared__ int s_slot[DP_WARPS][32];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int t = blockIdx.x * DP_WARPS + wl;
    if (t >= S) return;
    load_slots(s_slot[wl], slot_of, t, K, cap, lane, status);
    const int nunits = H >> 4, nb = H >> 7;
    constexpr int LOADS = IN_F32 ? 4 : 2;  // 16-byte loads per unit
    const uint8_t *src = reinterpret_cast<const uint8_t *>(x) + (size_t)t * H * (IN_F32 ? 4 : 2);
    for (int u0 = 0; u0 < nunits; u0 += 32 * UNROLL) {
        U4 raw[UNROLL][LOADS];
#pragma unroll
        for (int j = 0; j < UNROLL; ++j) {
            const int u = u0 + 32 * j + lane;
            if (u < nunits) {
#pragma unroll
                for (int l = 0; l < LOADS; ++l) raw[j][l] = ld_nc_v4(src + (size_t)u * 16 * LOADS + 16 * l);
            } else {
#pragma unroll
                for (int l = 0; l < LOADS; ++l) raw[j][l] = U4{0, 0, 0, 0};
            }
        }
        U4 q[UNROLL];
        float scale[UNROLL];
#pragma unroll
        for (int j = 0; j < UNROLL; ++j) {
            float f[16];
            if (IN_F32) {
#pragma unroll
                for (int l = 0; l < 4; ++l) {
                    f[4 * l + 0] = __uint_as_float(raw[j][l].x);
                    f[4 * l + 1] = __uint_as_float(raw[j][l].y);
                    f[4 * l + 2] = __uint_as_float(raw[j][l].z);
                    f[4 * l + 3] = __uint_as_float(raw[j][l].w);
                }
            } else {
#pragma unroll
                for (int l = 0; l < 2; ++l) {
                    f[8 * l + 0] = bf16lo(raw[j][l].x);
                    f[8 * l + 1] = bf16hi(raw[j][l].x);
                    f[8 * l + 2] = bf16lo(raw[j][l].y);
                    f[8 * l + 3] = bf16hi(raw[j][l].y);
                    f[8 * l + 4] = bf16lo(raw[j][l].z);
                    f[8 * l + 5] = bf16hi(raw[j][l].z);
                    f[8 * l + 6] = bf16lo(raw[j][l].w);
                    f[8 * l + 7] = bf16hi(raw[j][l].w);
                }
            }
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 4));
            const float s = __fdiv_rn(amax, 448.0f);
            scale[j] = s;
            q[j] = quant16(f, s);
        }
        for (int k = 0; k < K; ++k) {
            const int s = s_slot[wl][k];
            if (s < 0) continue;
            uint8_t *dst = xd + (size_t)s * H;
            float *sdst = xs + (size_t)s * nb;
#pragma unroll
            for (int j = 0; j < UNROLL; ++j) {
                const int u = u0 + 32 * j + lane;
                if (u < nunits) {
                    st_v4(dst + (size_t)u * 16, q[j]);
                    if ((lane & 7) == 0) sdst[u >> 3] = scale[j];
                }
            }
        }
    }
}

cudaError_t launch_dispatch(const void *x, int dtype, int S, int H, int K, const int32_t *slot_of,
                            int quant, void *xd, float *xs, int64_t cap, int32_t *status,
                            cudaStream_t st) {
    if (S == 0) return cudaSuccess;
    const int blocks = (S + DP_WARPS - 1) / DP_WARPS;
    if (quant == MOE_QUANT_NONE) {
        const int nunits = (int)(((size_t)H * (dtype == MOE_DTYPE_F32 ? 4 : 2)) / 16);
        dispatch_copy_kernel<2><<<blocks, DP_THREADS, 0, st>>>(
            reinterpret_cast<const uint8_t *>(x), S, nunits, K, slot_of,
            reinterpret_cast<uint8_t *>(xd), cap, status);
    } else if (dtype == MOE_DTYPE_BF16) {
        dispatch_fp8_kernel<false, 2><<<blocks, DP_THREADS, 0, st>>>(
            x, S, H, K, slot_of, reinterpret_cast<uint8_t *>(xd), xs, cap, status);
    } else {
        dispatch_fp8_kernel<true, 1><<<blocks, DP_THREADS, 0, st>>>(
            x, S, H, K, slot_of, reinterpret_cast<uint8_t *>(xd), xs, cap, status);
    }
    return cudaGetLastError();
}

}  // namespace moe
