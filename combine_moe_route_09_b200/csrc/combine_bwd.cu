// Backward of the combine with the dual-residual epilogue (training).
//
// "MoonEP developer guide", core API example: the backward pass reuses the
// plan built in the forward pass.  With g = dL/d(residual_out) and
// gn = dL/d(residual_no_routed_out), the forward
//     out = residual + (shared + sum_k w_k y_k),  rnr = residual + shared
// has, per token t and valid pair k,
//     grad_y[slot]  = w_k g            (fp32 product, rounded once)
//     grad_w[t, k]  = <y[slot], g>     (fp32 sum, fixed order)
//     grad_skip[t]  = g + gn           (the gradient of residual and of shared_out)
//
// Persistent kernel on the same pipeline as the forward combine: a producer
// warp bulk-loads, per (token, chunk) item, the K gathered y chunks, the g
// chunk and the gn chunk into a 2-stage ring (cp.async.bulk, mbarriers, no
// multicast); W consumer warps (4 for rows up to 2 KB, 6 up to 8 KB, 16 for
// longer rows) hold one 16-byte unit per thread.  Each CTA takes whole tokens, so grad_w needs no
// atomics: per item every warp reduces its dot-product partials with a fixed
// xor tree and lane k keeps pair k's running sum; at the token's last chunk the
// W warps' sums are added in warp order.  The reduction barrier there is an
// AND-barrier, so a timed-out wait makes all consumer warps leave together.
#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace moe {

// 2 stages.  Rows of at most 2 KB: 4 consumer warps with 2 KB chunks (about 42 KB
// a CTA, 5 CTAs an SM at K = 8).  Rows of at most 8 KB: 6 warps with 3 KB chunks
// (3 CTAs an SM).  Longer rows: 16 warps with 8 KB chunks (one CTA an SM).  A
// sweep of 4 to 16 consumer warps, 2 to 4 stages and 1 to 5 CTAs an SM found no
// single setting faster on every shape.  In the graph-replayed backward step
// (combine, dispatch and router backward): 16 warps took 4096 x 7168 from 282.4
// to 270.9 us, 6 warps took 16384 x 2048 from 357.9 to 311.1 us (10 warps:
// 311.2 us), while 4096 x 768 rows ran 19.5 us with 4 warps against 41 us with 16.
constexpr int BW_STAGES = 2;
constexpr int BW_HDR = 384;  // per stage: valid mask, the token's K weights (at 4), K slots (at 132)
constexpr int BW_SHORT_ROW = 2048;  // bytes: rows up to this take 4 consumer warps
constexpr int BW_LONG_ROW = 8192;   // bytes: rows up to this take 6 consumer warps, longer rows 16
template <int W>
struct BwShape {
    static constexpr int CONSUMERS = W * 32;
    static constexpr int THREADS = CONSUMERS + 32;  // + the producer warp
    static constexpr int MAX_CHUNK = CONSUMERS * 16;
    static constexpr int SMEM_BUDGET = W > 4 ? 200 * 1024 : 100 * 1024;  // ring bytes per CTA
};

struct CombineBwdArgs {
    const uint8_t *g, *gn, *y;
    const int32_t *slot_of;
    const float *topk_w;
    uint8_t *grad_y;
    float *grad_w;
    uint8_t *grad_skip;
    int32_t *status;
    int64_t cap;
    int S, K, row_bytes, chunk, nchunks;
};

template <bool F32>
struct BVec;

template <>
struct BVec<false> {
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
struct BVec<true> {
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

template <int W, bool F32, bool HAS_GN, bool HAS_SKIP>
__global__ void __launch_bounds__(BwShape<W>::THREADS) combine_bwd_kernel(const CombineBwdArgs a) {
    using V = BVec<F32>;
    constexpr int N = V::N;
    extern __shared__ __align__(128) uint8_t smem[];
    // [STAGES][header (mask, weights, slots) | K y chunks | g chunk | gn chunk] | barriers |
    // per-warp dot sums [2][4][32]
    const int K = a.K, chunk = a.chunk;
    const int stage_bytes = BW_HDR + (K + 2) * chunk;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + BW_STAGES * stage_bytes);
    float *wsum = reinterpret_cast<float *>(bars + 2 * BW_STAGES);
    const uint32_t smem0 = smem_addr(smem);
    const uint32_t bar0 = smem_addr(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (BW_STAGES + s); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < BW_STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), W);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    // whole tokens per CTA: [t_first, t_last)
    const int t_first = (int)((long long)a.S * blockIdx.x / gridDim.x);
    const int t_last = (int)((long long)a.S * (blockIdx.x + 1) / gridDim.x);
    const long long first = (long long)t_first * a.nchunks, last = (long long)t_last * a.nchunks;

    if (warp == W) {
        // ------------------------------- producer -------------------------------
        int t_cur = -1, cur = -1, nxt = -1;
        float cur_w = 0.f, nxt_w = 0.f;
        uint32_t valid = 0;
        if (first < last && lane < K) {
            nxt = __ldg(a.slot_of + (size_t)t_first * K + lane);
            nxt_w = __ldg(a.topk_w + (size_t)t_first * K + lane);
        }
        int i = 0;
        bool ok = true;
        int t = t_first, c = 0;
        for (long long item = first; item < last && ok; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
            const int s = i % BW_STAGES;
            if (t != t_cur) {
                t_cur = t;
                cur = nxt;
                cur_w = nxt_w;
                if ((int64_t)cur >= a.cap) {
                    set_status(a.status, MOE_STATUS_BAD_SLOT);
                    cur = -1;
                }
                valid = __ballot_sync(FULL, cur >= 0);
                if (lane < K && t + 1 < t_last) {
                    nxt = __ldg(a.slot_of + (size_t)(t + 1) * K + lane);
                    nxt_w = __ldg(a.topk_w + (size_t)(t + 1) * K + lane);
                }
            }
            if (i >= BW_STAGES)
                ok = __all_sync(FULL, mbar_wait(empty_bar(s), ((i / BW_STAGES) - 1) & 1, a.status));
            if (!ok) break;
            const int off = c * chunk;
            const uint32_t bytes = (uint32_t)min(chunk, a.row_bytes - off);
            const uint32_t stage = smem0 + (uint32_t)(s * stage_bytes);
            if (lane < K) {
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(stage + 4u + 4u * lane), "f"(cur_w) : "memory");
                asm volatile("st.shared.s32 [%0], %1;" ::"r"(stage + 132u + 4u * lane), "r"(cur) : "memory");
            }
            if (lane == 0) asm volatile("st.shared.u32 [%0], %1;" ::"r"(stage), "r"(valid) : "memory");
            __syncwarp();
            if (lane == 0) {
                const uint32_t n = (uint32_t)__popc(valid) + 1u + (HAS_GN ? 1u : 0u);
                mbar_arrive_expect_tx(full_bar(s), n * bytes);
            }
            __syncwarp();
            const uint32_t data = stage + BW_HDR;
            if (cur >= 0)
                bulk_g2s(data + (uint32_t)(lane * chunk), a.y + (size_t)cur * a.row_bytes + off, bytes, full_bar(s));
            const size_t tok = (size_t)t * a.row_bytes + off;
            if (lane == 0) bulk_g2s(data + (uint32_t)(K * chunk), a.g + tok, bytes, full_bar(s));
            if (HAS_GN && lane == 1) bulk_g2s(data + (uint32_t)((K + 1) * chunk), a.gn + tok, bytes, full_bar(s));
        }
        if (lane == 0) {
            for (int j = i - BW_STAGES; j < i; ++j)
                if (j >= 0) mbar_wait(full_bar(j % BW_STAGES), (j / BW_STAGES) & 1, a.status);
        }
        return;
    }

    // ------------------------------- consumers -------------------------------
    bool failed = false;  // a wait timed out: stop touching the ring, still meet the barriers
    float run = 0.f;      // lane k: this warp's running <y_k, g> of the current token
    int i = 0, t = t_first, c = 0, ntok = 0;
    for (long long item = first; item < last; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
        const int s = i % BW_STAGES;
        if (!failed) failed = !__all_sync(FULL, mbar_wait(full_bar(s), (i / BW_STAGES) & 1, a.status));
        if (!failed) {
            const int off = c * chunk;
            const int bytes = min(chunk, a.row_bytes - off);
            const uint32_t stage = smem0 + (uint32_t)(s * stage_bytes);
            const uint32_t data = stage + BW_HDR;
            uint32_t valid;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(valid) : "r"(stage) : "memory");
            const int ub = tid * 16;
            const bool active = ub < bytes;
            float gf[N] = {};
            if (active) V::unpack(lds128(data + (uint32_t)(K * chunk + ub)), gf);
            const size_t tok = (size_t)t * a.row_bytes + off + ub;
            if (HAS_SKIP && active) {
                float o[N];
                if (HAS_GN) {
                    float nf[N];
                    V::unpack(lds128(data + (uint32_t)((K + 1) * chunk + ub)), nf);
#pragma unroll
                    for (int e = 0; e < N; ++e) o[e] = __fadd_rn(gf[e], nf[e]);
                } else {
#pragma unroll
                    for (int e = 0; e < N; ++e) o[e] = gf[e];
                }
                st_v4(a.grad_skip + tok, V::pack(o));
            }
            for (int k = 0; k < K; ++k) {
                float p = 0.f;
                if ((valid >> k) & 1u) {
                    if (active) {
                        float wk;
                        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(wk) : "r"(stage + 4u + 4u * k) : "memory");
                        float yf[N], gy[N];
                        V::unpack(lds128(data + (uint32_t)(k * chunk + ub)), yf);
#pragma unroll
                        for (int e = 0; e < N; ++e) {
                            p = __fmaf_rn(yf[e], gf[e], p);
                            gy[e] = __fmul_rn(wk, gf[e]);
                        }
                        int sl;
                        asm volatile("ld.shared.s32 %0, [%1];" : "=r"(sl) : "r"(stage + 132u + 4u * k) : "memory");
                        st_v4(a.grad_y + (size_t)sl * a.row_bytes + off + ub, V::pack(gy));
                    }
                    // fixed xor tree: every lane ends with the warp's partial for pair k
#pragma unroll
                    for (int m = 16; m > 0; m >>= 1) p += __shfl_xor_sync(FULL, p, m);
                    if (lane == k) run += p;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));
        }
        if (c == a.nchunks - 1) {
            // token end: add the W warps' sums in warp order
            const int par = ntok & 1;
            if (lane < K) wsum[(par * W + warp) * 32 + lane] = run;
            if (!named_bar_and(1, BwShape<W>::CONSUMERS, !failed)) break;
            if (warp == 0 && lane < K) {
                float sum = 0.f;
#pragma unroll
                for (int ww = 0; ww < W; ++ww)
                    sum = __fadd_rn(sum, wsum[(par * W + ww) * 32 + lane]);
                a.grad_w[(size_t)t * K + lane] = sum;
            }
            run = 0.f;
            ++ntok;
        }
    }
}

template <int W, bool F32, bool GN, bool SKIP>
static cudaError_t launch_bwd(CombineBwdArgs a, cudaStream_t st) {
    auto kern = combine_bwd_kernel<W, F32, GN, SKIP>;
    int chunk = BwShape<W>::MAX_CHUNK;
    while (chunk > 256 && BW_STAGES * (BW_HDR + (a.K + 2) * chunk) > BwShape<W>::SMEM_BUDGET) chunk >>= 1;
    a.chunk = chunk < a.row_bytes ? chunk : a.row_bytes;
    a.nchunks = (a.row_bytes + a.chunk - 1) / a.chunk;
    const size_t smem = (size_t)BW_STAGES * (BW_HDR + (a.K + 2) * a.chunk) + 2 * BW_STAGES * 8 +
                        2 * W * 32 * sizeof(float);
    static KernelSlots<decltype(kern)> slots;
    int sms = 0, per_sm = 0;
    cudaError_t e = slots.prepare(kern, BwShape<W>::THREADS, smem, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    long long grid = (long long)sms * per_sm;
    if (grid > a.S) grid = a.S;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(BwShape<W>::THREADS), smem, st, a);
}

template <int W, bool F32>
static cudaError_t launch_bwd_dt(const CombineBwdArgs &a, cudaStream_t st) {
    const bool gn = a.gn, skip = a.grad_skip;
    if (gn && skip) return launch_bwd<W, F32, true, true>(a, st);
    if (gn) return launch_bwd<W, F32, true, false>(a, st);
    if (skip) return launch_bwd<W, F32, false, true>(a, st);
    return launch_bwd<W, F32, false, false>(a, st);
}

cudaError_t launch_combine_backward(const void *g, const void *gn, const void *y, int dtype, int S, int H,
                                    int K, int64_t cap, const int32_t *slot_of, const float *topk_w,
                                    void *grad_y, float *grad_w, void *grad_skip, int32_t *status,
                                    cudaStream_t st) {
    if (S == 0) return cudaSuccess;
    const bool f32 = dtype == MOE_DTYPE_F32;
    CombineBwdArgs a;
    a.g = reinterpret_cast<const uint8_t *>(g);
    a.gn = reinterpret_cast<const uint8_t *>(gn);
    a.y = reinterpret_cast<const uint8_t *>(y);
    a.slot_of = slot_of;
    a.topk_w = topk_w;
    a.grad_y = reinterpret_cast<uint8_t *>(grad_y);
    a.grad_w = grad_w;
    a.grad_skip = reinterpret_cast<uint8_t *>(grad_skip);
    a.status = status;
    a.cap = cap;
    a.S = S;
    a.K = K;
    a.row_bytes = H * (f32 ? 4 : 2);
    if (a.row_bytes > BW_LONG_ROW) return f32 ? launch_bwd_dt<16, true>(a, st) : launch_bwd_dt<16, false>(a, st);
    if (a.row_bytes > BW_SHORT_ROW) return f32 ? launch_bwd_dt<6, true>(a, st) : launch_bwd_dt<6, false>(a, st);
    return f32 ? launch_bwd_dt<4, true>(a, st) : launch_bwd_dt<4, false>(a, st);
}

}  // namespace moe
