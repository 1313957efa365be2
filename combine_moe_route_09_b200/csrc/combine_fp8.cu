// Combine over FP8 expert outputs: e4m3 rows with one fp32 scale per 128
// channels (the format the FP8 dispatch produces; "Efficient and portable
// mixture-of-experts communication", Dispatch: tokens travel with their block
// scaling factors), gathered, dequantised (y = e4m3_value * scale, an fp32
// product), weighted and accumulated in fp32 in ascending k, with the same
// dual-residual epilogue as the bf16/fp32 combine.  Reading one byte per
// gathered element instead of two halves the dominant traffic.
//
// Same persistent, warp-specialised pipeline as combine.cu: a producer warp
// bulk-loads, per (token, chunk) item, the K code chunks and the K matching
// scale segments (cp.async.bulk; H % 512 == 0 keeps every scale segment
// 16-byte aligned), plus the shared_out and residual chunks, into a 4-stage
// ring; 4 consumer warps take 8 channels per thread.
#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace moe {

constexpr int C8_STAGES = 4;
constexpr int C8_CONSUMER_WARPS = 4;
constexpr int C8_CONSUMERS = C8_CONSUMER_WARPS * 32;
constexpr int C8_THREADS = C8_CONSUMERS + 32;
constexpr int C8_HDR = 256;  // per stage: valid mask, then the token's K weights

struct CombineFp8Args {
    const uint8_t *yq;      // [cap, H] e4m3
    const float *ys;        // [cap, H / 128]
    const int32_t *slot_of;
    const float *topk_w;
    const uint8_t *shared_out;
    const uint8_t *residual;  // may alias out
    uint8_t *out;
    uint8_t *out_no_routed;
    int32_t *status;
    int64_t cap;
    int S, H, K;
    int ob;      // output element bytes (2 or 4)
    int cch;     // channels per item (512 or 1024)
    int nchunks;
};

__device__ __forceinline__ float half_bits_to_f32(uint32_t h) {
    float f;
    asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"((unsigned short)h));
    return f;
}

// 8 e4m3 codes (two 32-bit words, code i in byte i) -> 8 floats (exact: every
// e4m3 value is an f16 value, and every f16 value an f32 value).
__device__ __forceinline__ void decode8(uint32_t lo, uint32_t hi, float (&f)[8]) {
    const uint32_t w[2] = {lo, hi};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint16_t pair = (uint16_t)(w[i] >> (16 * j));
            uint32_t h2;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
            f[4 * i + 2 * j + 0] = half_bits_to_f32(h2 & 0xffffu);
            f[4 * i + 2 * j + 1] = half_bits_to_f32(h2 >> 16);
        }
    }
}

// KT: K known at compile time (0 = runtime K); with it the per-pair loop unrolls.
template <bool F32, bool HAS_SH, bool HAS_RS, bool HAS_RNR, int KT>
__global__ void __launch_bounds__(C8_THREADS) combine_fp8_kernel(const CombineFp8Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    // [STAGES][header | K code chunks (cch B) | K scale segments (cch/32 B) | shared | residual]
    const int K = KT > 0 ? KT : a.K, cch = a.cch;
    const int seg = cch / 32;  // scale bytes per item and row
    const int obytes = cch * a.ob;
    const int stage_bytes = C8_HDR + K * cch + K * seg + 2 * obytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C8_STAGES * stage_bytes);
    const uint32_t smem0 = smem_addr(smem);
    const uint32_t bar0 = smem_addr(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C8_STAGES + s); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < C8_STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), C8_CONSUMER_WARPS);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    const long long nitems = (long long)a.S * a.nchunks;
    const long long first = nitems * blockIdx.x / gridDim.x;
    const long long last = nitems * (blockIdx.x + 1) / gridDim.x;
    const int nb = a.H >> 7;
    const int row_out = a.H * a.ob;
    if (warp == C8_CONSUMER_WARPS) {
        // ------------------------------- producer -------------------------------
        int t_cur = -1, cur = -1, nxt = -1;
        float cur_w = 0.f, nxt_w = 0.f;
        uint32_t valid = 0;
        if (first < last && lane < K) {
            const size_t o = (size_t)(first / a.nchunks) * K + lane;
            nxt = __ldg(a.slot_of + o);
            nxt_w = __ldg(a.topk_w + o);
        }
        int i = 0;
        bool ok = true;
        int t = (int)(first / a.nchunks), c = (int)(first - (long long)t * a.nchunks);
        for (long long item = first; item < last && ok; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
            const int s = i % C8_STAGES;
            if (t != t_cur) {
                t_cur = t;
                cur = nxt;
                cur_w = nxt_w;
                if ((int64_t)cur >= a.cap) {
                    set_status(a.status, MOE_STATUS_BAD_SLOT);
                    cur = -1;
                }
                valid = __ballot_sync(FULL, cur >= 0);
                if (lane < K && (long long)(t + 1) * a.nchunks < last) {
                    nxt = __ldg(a.slot_of + (size_t)(t + 1) * K + lane);
                    nxt_w = __ldg(a.topk_w + (size_t)(t + 1) * K + lane);
                }
            }
            if (i >= C8_STAGES)
                ok = __all_sync(FULL, mbar_wait(empty_bar(s), ((i / C8_STAGES) - 1) & 1, a.status));
            if (!ok) break;
            const int col0 = c * cch;
            const uint32_t stage = smem0 + (uint32_t)(s * stage_bytes);
            if (lane < K)
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(stage + 4u + 4u * lane), "f"(cur_w) : "memory");
            if (lane == 0) asm volatile("st.shared.u32 [%0], %1;" ::"r"(stage), "r"(valid) : "memory");
            __syncwarp();
            if (lane == 0) {
                const uint32_t n = (uint32_t)__popc(valid);
                mbar_arrive_expect_tx(full_bar(s), n * (uint32_t)(cch + seg) +
                                                       ((HAS_SH ? 1u : 0u) + (HAS_RS ? 1u : 0u)) * (uint32_t)obytes);
            }
            __syncwarp();
            const uint32_t data = stage + C8_HDR;
            if (cur >= 0) {
                bulk_g2s(data + (uint32_t)(lane * cch), a.yq + (size_t)cur * a.H + col0, (uint32_t)cch, full_bar(s));
                bulk_g2s(data + (uint32_t)(K * cch + lane * seg), a.ys + (size_t)cur * nb + (col0 >> 7),
                         (uint32_t)seg, full_bar(s));
            }
            const size_t tok = (size_t)t * row_out + (size_t)col0 * a.ob;
            const uint32_t sd = data + (uint32_t)(K * (cch + seg));
            if (HAS_SH && lane == 0) bulk_g2s(sd, a.shared_out + tok, (uint32_t)obytes, full_bar(s));
            if (HAS_RS && lane == 1) bulk_g2s(sd + (uint32_t)obytes, a.residual + tok, (uint32_t)obytes, full_bar(s));
        }
        if (lane == 0) {
            for (int j = i - C8_STAGES; j < i; ++j)
                if (j >= 0) mbar_wait(full_bar(j % C8_STAGES), (j / C8_STAGES) & 1, a.status);
        }
        return;
    }

    // ------------------------------- consumers -------------------------------
    // Thread tid: channels [8 tid, 8 tid + 8) of the item (its block: tid / 16).
    int i = 0;
    int t = (int)(first / a.nchunks), c = (int)(first - (long long)t * a.nchunks);
    for (long long item = first; item < last; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
        const int s = i % C8_STAGES;
        if (!__all_sync(FULL, mbar_wait(full_bar(s), (i / C8_STAGES) & 1, a.status))) break;
        const uint32_t stage = smem0 + (uint32_t)(s * stage_bytes);
        const uint32_t data = stage + C8_HDR;
        uint32_t valid;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(valid) : "r"(stage) : "memory");
        const int ch = tid * 8;
        if (ch < cch) {
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
            constexpr int KU = KT > 0 ? KT : 1;
#pragma unroll(KU)
            for (int k = 0; k < K; ++k) {
                if (!((valid >> k) & 1u)) continue;
                float wk, sc;
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(wk) : "r"(stage + 4u + 4u * k) : "memory");
                asm volatile("ld.shared.f32 %0, [%1];"
                             : "=f"(sc)
                             : "r"(data + (uint32_t)(K * cch + k * seg + (ch >> 7) * 4))
                             : "memory");
                uint32_t q0, q1;
                asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                             : "=r"(q0), "=r"(q1)
                             : "r"(data + (uint32_t)(k * cch + ch))
                             : "memory");
                float f[8];
                decode8(q0, q1, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(wk, __fmul_rn(f[e], sc), acc[e]);
            }
            const uint32_t sd = data + (uint32_t)(K * (cch + seg)) + (uint32_t)(ch * a.ob);
            float fsh[8] = {}, frs[8] = {}, o[8];
            if (F32) {
                if (HAS_SH) {
                    const U4 v0 = lds128(sd), v1 = lds128(sd + 16u);
                    fsh[0] = __uint_as_float(v0.x); fsh[1] = __uint_as_float(v0.y);
                    fsh[2] = __uint_as_float(v0.z); fsh[3] = __uint_as_float(v0.w);
                    fsh[4] = __uint_as_float(v1.x); fsh[5] = __uint_as_float(v1.y);
                    fsh[6] = __uint_as_float(v1.z); fsh[7] = __uint_as_float(v1.w);
                }
                if (HAS_RS) {
                    const U4 v0 = lds128(sd + (uint32_t)obytes), v1 = lds128(sd + (uint32_t)obytes + 16u);
                    frs[0] = __uint_as_float(v0.x); frs[1] = __uint_as_float(v0.y);
                    frs[2] = __uint_as_float(v0.z); frs[3] = __uint_as_float(v0.w);
                    frs[4] = __uint_as_float(v1.x); frs[5] = __uint_as_float(v1.y);
                    frs[6] = __uint_as_float(v1.z); frs[7] = __uint_as_float(v1.w);
                }
            } else {
                if (HAS_SH) {
                    const U4 v = lds128(sd);
                    fsh[0] = bf16lo(v.x); fsh[1] = bf16hi(v.x); fsh[2] = bf16lo(v.y); fsh[3] = bf16hi(v.y);
                    fsh[4] = bf16lo(v.z); fsh[5] = bf16hi(v.z); fsh[6] = bf16lo(v.w); fsh[7] = bf16hi(v.w);
                }
                if (HAS_RS) {
                    const U4 v = lds128(sd + (uint32_t)obytes);
                    frs[0] = bf16lo(v.x); frs[1] = bf16hi(v.x); frs[2] = bf16lo(v.y); frs[3] = bf16hi(v.y);
                    frs[4] = bf16lo(v.z); frs[5] = bf16hi(v.z); frs[6] = bf16lo(v.w); frs[7] = bf16hi(v.w);
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float m = acc[e];
                if (HAS_SH) m = __fadd_rn(fsh[e], m);
                o[e] = HAS_RS ? __fadd_rn(frs[e], m) : m;
            }
            const size_t g = (size_t)t * row_out + (size_t)(c * cch + ch) * a.ob;
            float n[8];
            if (HAS_RNR) {
#pragma unroll
                for (int e = 0; e < 8; ++e) n[e] = __fadd_rn(frs[e], fsh[e]);
            }
            if (F32) {
                st_v4(a.out + g, U4{__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                                    __float_as_uint(o[3])});
                st_v4(a.out + g + 16, U4{__float_as_uint(o[4]), __float_as_uint(o[5]), __float_as_uint(o[6]),
                                         __float_as_uint(o[7])});
                if (HAS_RNR) {
                    st_v4(a.out_no_routed + g, U4{__float_as_uint(n[0]), __float_as_uint(n[1]),
                                                  __float_as_uint(n[2]), __float_as_uint(n[3])});
                    st_v4(a.out_no_routed + g + 16, U4{__float_as_uint(n[4]), __float_as_uint(n[5]),
                                                       __float_as_uint(n[6]), __float_as_uint(n[7])});
                }
            } else {
                st_v4(a.out + g, U4{pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                    pack_bf16x2(o[6], o[7])});
                if (HAS_RNR)
                    st_v4(a.out_no_routed + g, U4{pack_bf16x2(n[0], n[1]), pack_bf16x2(n[2], n[3]),
                                                  pack_bf16x2(n[4], n[5]), pack_bf16x2(n[6], n[7])});
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
    }
}

template <bool F32, bool SH, bool RS, bool RNR>
static cudaError_t launch_c8(const CombineFp8Args &a, cudaStream_t st) {
    auto kern = a.K == 8 ? combine_fp8_kernel<F32, SH, RS, RNR, 8> : combine_fp8_kernel<F32, SH, RS, RNR, 0>;
    const int seg = a.cch / 32;
    const size_t smem = (size_t)C8_STAGES * (C8_HDR + a.K * (a.cch + seg) + 2 * a.cch * a.ob) + 2 * C8_STAGES * 8;
    static KernelSlots<decltype(kern)> slots;
    int sms = 0, per_sm = 0;
    cudaError_t e = slots.prepare(kern, C8_THREADS, smem, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    const long long nitems = (long long)a.S * a.nchunks;
    long long grid = (long long)sms * per_sm;
    if (grid > nitems) grid = nitems;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(C8_THREADS), smem, st, a);
}

template <bool F32>
static cudaError_t launch_c8_dt(const CombineFp8Args &a, cudaStream_t st) {
    const bool sh = a.shared_out, rs = a.residual, rnr = a.out_no_routed;
    if (sh && rs && rnr) return launch_c8<F32, true, true, true>(a, st);
    if (sh && rs) return launch_c8<F32, true, true, false>(a, st);
    if (sh) return launch_c8<F32, true, false, false>(a, st);
    if (rs) return launch_c8<F32, false, true, false>(a, st);
    return launch_c8<F32, false, false, false>(a, st);
}

cudaError_t launch_combine_fp8(const uint8_t *yq, const float *ys, int dtype, int S, int H, int K, int64_t cap,
                               const int32_t *slot_of, const float *topk_w, const void *shared_out,
                               const void *residual, void *out, void *out_no_routed, int32_t *status,
                               cudaStream_t st) {
    if (S == 0) return cudaSuccess;
    const bool f32 = dtype == MOE_DTYPE_F32;
    CombineFp8Args a;
    a.yq = yq;
    a.ys = ys;
    a.slot_of = slot_of;
    a.topk_w = topk_w;
    a.shared_out = reinterpret_cast<const uint8_t *>(shared_out);
    a.residual = reinterpret_cast<const uint8_t *>(residual);
    a.out = reinterpret_cast<uint8_t *>(out);
    a.out_no_routed = reinterpret_cast<uint8_t *>(out_no_routed);
    a.status = status;
    a.cap = cap;
    a.S = S;
    a.H = H;
    a.K = K;
    a.ob = f32 ? 4 : 2;
    a.cch = (H % 1024 == 0 && K <= 16) ? 1024 : 512;
    a.nchunks = H / a.cch;
    return f32 ? launch_c8_dt<true>(a, st) : launch_c8_dt<false>(a, st);
}

}  // namespace moe
