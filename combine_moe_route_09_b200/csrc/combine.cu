// Combine: gather each token's K expert-output rows, take the router-weighted
// sum in fp32, and fuse the FarSkip-Collective dual-residual epilogue.
//
// "Efficient and portable mixture-of-experts communication", Combine: the
// receiver reads the payloads the routing table names and averages them with
// the router's weights.  Instella-MoE / FarSkip-Collective explainer, the dual
// residual stream:  residual_no_routed = residual + shared_out;
//                   residual = residual + (shared_out + routed).
//
// One warp per token, 16-byte units.  For each unit a lane issues all K
// gathered loads plus the shared/residual loads before any arithmetic, then
// accumulates acc = fma(w_k, y_k, acc) in ascending k, adds shared, then
// residual, and rounds once to the output type.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int CB_THREADS = 256;
constexpr int CB_WARPS = CB_THREADS / 32;
constexpr int CB_KCHUNK = 8;  // gathered rows in flight per lane per unit

template <bool F32>
struct Vec;

template <>
struct Vec<false> {  // bf16: 8 elements per 16 bytes
    static constexpr int N = 8;
    __device__ static void unpack(const U4 &v, float (&f)[8]) {
        f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
        f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
    }
    __device__ static U4 pack(const float (&f)[8]) {
        return U4{pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                  pack_bf16x2(f[6], f[7])};
    }
};

template <>
struct Vec<true> {  // fp32: 4 elements per 16 bytes
    static constexpr int N = 4;
    __device__ static void unpack(const U4 &v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    __device__ static U4 pack(const float (&f)[4]) {
        return U4{__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                  __float_as_uint(f[3])};
    }
};

template <bool F32, bool HAS_SH, bool HAS_RS, bool HAS_RNR>
__global__ void __launch_bounds__(CB_THREADS)
    combine_kernel(const uint8_t *__restrict__ y, int S, int nunits, int K, int64_t cap,
                   const int32_t *__restrict__ slot_of, const float *__restrict__ topk_w,
                   const uint8_t *__restrict__ shared_out, const uint8_t *residual, uint8_t *out,
                   uint8_t *__restrict__ out_no_routed, int32_t *status) {
    using V = Vec<F32>;
    constexpr int N = V::N;
    __shared__ int s_slot[CB_WARPS][32];
    __shared__ float s_w[CB_WARPS][32];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int t = blockIdx.x * CB_WARPS + wl;
    if (t >= S) return;
    if (lane < K) {
        int s = __ldg(slot_of + (size_t)t * K + lane);
        if ((int64_t)s >= cap) {
            set_status(status, MOE_STATUS_BAD_SLOT);
            s = -1;
        }
        s_slot[wl][lane] = s;
        s_w[wl][lane] = __ldg(topk_w + (size_t)t * K + lane);
    }
    __syncwarp();
    const size_t row_bytes = (size_t)nunits * 16;
    const size_t tok = (size_t)t * row_bytes;
    for (int u = lane; u < nunits; u += 32) {
        const size_t ub = (size_t)u * 16;
        U4 sh, rs;
        if (HAS_SH) sh = ld_nc_v4(shared_out + tok + ub);
        if (HAS_RS) rs = *reinterpret_cast<const U4 *>(residual + tok + ub);  // may alias out
        float acc[N];
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] = 0.f;
        for (int k0 = 0; k0 < K; k0 += CB_KCHUNK) {
            U4 v[CB_KCHUNK];
#pragma unroll
            for (int kk = 0; kk < CB_KCHUNK; ++kk) {
                const int k = k0 + kk;
                const int s = k < K ? s_slot[wl][k] : -1;
                if (s >= 0) v[kk] = ld_nc_v4(y + (size_t)s * row_bytes + ub);
            }
#pragma unroll
            for (int kk = 0; kk < CB_KCHUNK; ++kk) {
                const int k = k0 + kk;
                const int s = k < K ? s_slot[wl][k] : -1;
                if (s >= 0) {
                    const float wk = s_w[wl][k];
                    float f[N];
                    V::unpack(v[kk], f);
#pragma unroll
                    for (int i = 0; i < N; ++i) acc[i] = __fmaf_rn(wk, f[i], acc[i]);
                }
            }
        }
        float fsh[N], frs[N], o[N];
        if (HAS_SH) V::unpack(sh, fsh);
        if (HAS_RS) V::unpack(rs, frs);
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float m = acc[i];
            if (HAS_SH) m = __fadd_rn(fsh[i], m);
            o[i] = HAS_RS ? __fadd_rn(frs[i], m) : m;
        }
        st_v4(out + tok + ub, V::pack(o));
        if (HAS_RNR) {
            float n[N];
#pragma unroll
            for (int i = 0; i < N; ++i) n[i] = __fadd_rn(frs[i], fsh[i]);
            st_v4(out_no_routed + tok + ub, V::pack(n));
        }
    }
}

template <bool F32, bool SH, bool RS, bool RNR>
static void launch_cb(const void *y, int S, int nunits, int K, int64_t cap, const int32_t *slot_of,
                      const float *w, const void *sh, const void *rs, void *out, void *rnr,
                      int32_t *status, cudaStream_t st) {
    const int blocks = (S + CB_WARPS - 1) / CB_WARPS;
    combine_kernel<F32, SH, RS, RNR><<<blocks, CB_THREADS, 0, st>>>(
        reinterpret_cast<const uint8_t *>(y), S, nunits, K, cap, slot_of, w,
        reinterpret_cast<const uint8_t *>(sh), reinterpret_cast<const uint8_t *>(rs),
        reinterpret_cast<uint8_t *>(out), reinterpret_cast<uint8_t *>(rnr), status);
}

template <bool F32>
static void launch_cb_dt(const void *y, int S, int nunits, int K, int64_t cap,
                         const int32_t *slot_of, const float *w, const void *sh, const void *rs,
                         void *out, void *rnr, int32_t *status, cudaStream_t st) {
    if (sh && rs && rnr)
        launch_cb<F32, true, true, true>(y, S, nunits, K, cap, slot_of, w, sh, rs, out, rnr, status, st);
    else if (sh && rs)
        launch_cb<F32, true, true, false>(y, S, nunits, K, cap, slot_of, w, sh, rs, out, rnr, status, st);
    else if (sh)
        launch_cb<F32, true, false, false>(y, S, nunits, K, cap, slot_of, w, sh, rs, out, rnr, status, st);
    else if (rs)
        launch_cb<F32, false, true, false>(y, S, nunits, K, cap, slot_of, w, sh, rs, out, rnr, status, st);
    else
        launch_cb<F32, false, false, false>(y, S, nunits, K, cap, slot_of, w, sh, rs, out, rnr, status, st);
}

cudaError_t launch_combine(const void *y, int dtype, int S, int H, int K, int64_t cap,
                           const int32_t *slot_of, const float *topk_w, const void *shared_out,
                           const void *residual, void *out, void *out_no_routed, int32_t *status,
                           cudaStream_t st) {
    if (S == 0) return cudaSuccess;
    const bool f32 = dtype == MOE_DTYPE_F32;
    const int nunits = (int)(((size_t)H * (f32 ? 4 : 2)) / 16);
    if (f32)
        launch_cb_dt<true>(y, S, nunits, K, cap, slot_of, topk_w, shared_out, residual, out,
                           out_no_routed, status, st);
    else
        launch_cb_dt<false>(y, S, nunits, K, cap, slot_of, topk_w, shared_out, residual, out,
                            out_no_routed, status, st);
    return cudaGetLastError();
}

}  // namespace moe
