// Combine: gather each token's K expert-output rows, take the router-weighted
// sum in fp32, and fuse the FarSkip-Collective dual-residual epilogue.
//
// "Efficient and portable mixture-of-experts communication", Combine: the
// receiver reads the payloads the routing table names and averages them with
// the router's weights.  Instella-MoE / FarSkip-Collective explainer, the dual
// residual stream:  residual_no_routed = residual + shared_out;
//                   residual = residual + (shared_out + routed).
//
// Persistent, warp-specialised kernel.  A work item is one column chunk
// (`chunk` bytes) of one token; each CTA of a grid sized to the resident CTA
// count takes a contiguous, balanced share of the items.
//   producer warp   per token: its K slots and weights (loaded one token
//                   ahead); per item: the valid mask and weights into the
//                   stage header, then one TMA bulk copy (cp.async.bulk
//                   global->shared, completing on the stage's mbarrier) per
//                   valid slot, plus the shared_out and residual chunks, into
//                   a ring of STAGES shared-memory stages.  No tensor maps,
//                   no multicast.
//   6 or 8 consumer warps per item: one 16-byte unit per thread; acc = fma(w_k, y_k,
//                   acc) in ascending k from shared memory, + shared, +
//                   residual, round once, 16-byte stores of both streams;
//                   then release the stage.
// HBM sees each gathered row chunk, shared_out and residual read once and both
// outputs written once.  All mbarrier waits are time-bounded.
#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace moe {

// W consumer warps take chunks of W * 512 bytes (one 16-byte unit per thread)
// through a 2-stage ring.  Rows of 2 to 8 KB take 6 warps (3 KB chunks, three
// CTAs per SM); the others take 8 warps (4 KB chunks, 82 KB per CTA with K = 8,
// two CTAs per SM).  On the DeepSeek-V3-shaped prefill combine 8 warps ran
// 107.0 us against 110.9 us for 4 warps with 2 KB chunks in 4 stages; 3 or 4
// stages of 4 KB, and 6 or 8 stages of smaller chunks, were slower.  On the
// 16384 x 2048 workload's 4 KB rows 6 warps took the step from 256.7 to
// 252.7 us (10 or 12 warps: 254.8 us); on rows of at most 2 KB, 4 warps, fast
// alone, lost in the step.
constexpr int CB_STAGES = 2;
constexpr int CB_SMEM_BUDGET = 100 * 1024;
constexpr int CB_MID_WARPS = 6;  // consumer warps for rows of 2 to 8 KB; 8 for the others
template <int W>
struct CbShape {
    static constexpr int CONSUMERS = W * 32;
    static constexpr int THREADS = CONSUMERS + 32;  // + the producer warp
    static constexpr int MAX_CHUNK = CONSUMERS * 16;
};

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

struct CombineArgs {
    const uint8_t *y;
    const int32_t *slot_of;
    const float *topk_w;
    const uint8_t *shared_out;
    const uint8_t *residual;  // may alias out
    uint8_t *out;
    uint8_t *out_no_routed;
    int32_t *status;
    int64_t cap;
    int S, K;
    int row_bytes;  // H * element size, a multiple of 16
    int chunk;      // bytes per work item, a multiple of 16, <= CbShape<W>::MAX_CHUNK
    int nchunks;    // ceil(row_bytes / chunk)
};

constexpr int CB_HDR = 256;  // per-stage header: valid mask, then the token's K weights

template <int W, bool F32, bool HAS_SH, bool HAS_RS, bool HAS_RNR>
__global__ void __launch_bounds__(CbShape<W>::THREADS) combine_kernel(const CombineArgs a) {
    using V = Vec<F32>;
    constexpr int N = V::N;
    extern __shared__ __align__(128) uint8_t smem[];
    // [STAGES][header | (K + 2) chunks: K gathered rows, shared_out, residual], then
    // the full / empty mbarriers of every stage
    const int K = a.K, chunk = a.chunk;
    const int stage_bytes = CB_HDR + (K + 2) * chunk;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + CB_STAGES * stage_bytes);
    const uint32_t smem0 = smem_addr(smem);
    const uint32_t bar0 = smem_addr(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (CB_STAGES + s); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < CB_STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), W);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    // This CTA's items: a contiguous, balanced share, so consecutive items
    // mostly belong to one token.
    const long long nitems = (long long)a.S * a.nchunks;
    const long long first = nitems * blockIdx.x / gridDim.x;
    const long long last = nitems * (blockIdx.x + 1) / gridDim.x;
    if (warp == W) {
        // ------------------------------- producer -------------------------------
        // Lane k holds the token's slot k and weight k, loaded one token ahead.
        int t_cur = -1, cur = -1, nxt = -1;
        float cur_w = 0.f, nxt_w = 0.f;
        uint32_t valid = 0;
        if (first < last && lane < K) {
            const size_t o = (size_t)(first / a.nchunks) * K + lane;
            nxt = __ldg(a.slot_of + o);
            nxt_w = a.topk_w ? __ldg(a.topk_w + o) : 1.0f;  // no weights: plain sum (dispatch backward)
        }
        int i = 0;
        bool ok = true;
        int t = (int)(first / a.nchunks), c = (int)(first - (long long)t * a.nchunks);
        for (long long item = first; item < last && ok; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
            const int s = i % CB_STAGES;
            if (t != t_cur) {
                t_cur = t;
                cur = nxt;
                cur_w = nxt_w;
                if ((int64_t)cur >= a.cap) {
                    set_status(a.status, MOE_STATUS_BAD_SLOT);
                    cur = -1;
                }
                valid = __ballot_sync(FULL, cur >= 0);
                const int tn = t + 1;
                if (lane < K && (long long)tn * a.nchunks < last) {
                    nxt = __ldg(a.slot_of + (size_t)tn * K + lane);
                    nxt_w = a.topk_w ? __ldg(a.topk_w + (size_t)tn * K + lane) : 1.0f;
                }
            }
            if (i >= CB_STAGES)
                ok = __all_sync(FULL, mbar_wait(empty_bar(s), ((i / CB_STAGES) - 1) & 1, a.status));
            if (!ok) break;
            const int off = c * chunk;
            const uint32_t bytes = (uint32_t)min(chunk, a.row_bytes - off);
            const uint32_t stage = smem0 + (uint32_t)(s * stage_bytes);
            if (lane < K)
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(stage + 4u + 4u * lane), "f"(cur_w) : "memory");
            if (lane == 0) asm volatile("st.shared.u32 [%0], %1;" ::"r"(stage), "r"(valid) : "memory");
            __syncwarp();
            if (lane == 0) {
                const uint32_t n = (uint32_t)__popc(valid) + (HAS_SH ? 1u : 0u) + (HAS_RS ? 1u : 0u);
                mbar_arrive_expect_tx(full_bar(s), n * bytes);
            }
            __syncwarp();
            const uint32_t data = stage + CB_HDR;
            if (cur >= 0)
                bulk_g2s(data + (uint32_t)(lane * chunk), a.y + (size_t)cur * a.row_bytes + off, bytes, full_bar(s));
            const size_t tok = (size_t)t * a.row_bytes + off;
            if (HAS_SH && lane == 0)
                bulk_g2s(data + (uint32_t)(K * chunk), a.shared_out + tok, bytes, full_bar(s));
            if (HAS_RS && lane == 1)
                bulk_g2s(data + (uint32_t)((K + 1) * chunk), a.residual + tok, bytes, full_bar(s));
        }
        // Never leave copies in flight: wait (bounded) for every stage still loading.
        if (lane == 0) {
            for (int j = i - CB_STAGES; j < i; ++j)
                if (j >= 0) mbar_wait(full_bar(j % CB_STAGES), (j / CB_STAGES) & 1, a.status);
        }
        return;
    }

    // ------------------------------- consumers -------------------------------
    int i = 0;
    int t = (int)(first / a.nchunks), c = (int)(first - (long long)t * a.nchunks);
    for (long long item = first; item < last; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
        const int s = i % CB_STAGES;
        if (!__all_sync(FULL, mbar_wait(full_bar(s), (i / CB_STAGES) & 1, a.status))) break;
        const int off = c * chunk;
        const int bytes = min(chunk, a.row_bytes - off);
        const uint32_t stage = smem0 + (uint32_t)(s * stage_bytes);
        const uint32_t data = stage + CB_HDR;
        uint32_t valid;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(valid) : "r"(stage) : "memory");
        const int ub = tid * 16;
        if (ub < bytes) {
            float acc[N];
#pragma unroll
            for (int e = 0; e < N; ++e) acc[e] = 0.f;
            for (int k = 0; k < K; ++k) {
                if (!((valid >> k) & 1u)) continue;
                float wk;
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(wk) : "r"(stage + 4u + 4u * k) : "memory");
                float f[N];
                V::unpack(lds128(data + (uint32_t)(k * chunk + ub)), f);
#pragma unroll
                for (int e = 0; e < N; ++e) acc[e] = __fmaf_rn(wk, f[e], acc[e]);
            }
            float fsh[N] = {}, frs[N] = {}, o[N];
            if (HAS_SH) V::unpack(lds128(data + (uint32_t)(K * chunk + ub)), fsh);
            if (HAS_RS) V::unpack(lds128(data + (uint32_t)((K + 1) * chunk + ub)), frs);
#pragma unroll
            for (int e = 0; e < N; ++e) {
                float m = acc[e];
                if (HAS_SH) m = __fadd_rn(fsh[e], m);
                o[e] = HAS_RS ? __fadd_rn(frs[e], m) : m;
            }
            const size_t g = (size_t)t * a.row_bytes + off + ub;
            st_v4(a.out + g, V::pack(o));
            if (HAS_RNR) {
                float n[N];
#pragma unroll
                for (int e = 0; e < N; ++e) n[e] = __fadd_rn(frs[e], fsh[e]);
                st_v4(a.out_no_routed + g, V::pack(n));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
    }
}

template <int W>
static int combine_chunk(int K, int row_bytes) {
    int chunk = CbShape<W>::MAX_CHUNK;
    while (chunk > 256 && CB_STAGES * (CB_HDR + (K + 2) * chunk) > CB_SMEM_BUDGET) chunk >>= 1;
    return chunk < row_bytes ? chunk : row_bytes;
}

static size_t combine_smem(int K, int chunk) {
    return (size_t)CB_STAGES * (CB_HDR + (K + 2) * chunk) + 2 * CB_STAGES * 8;
}

template <int W, bool F32, bool SH, bool RS, bool RNR>
static cudaError_t launch_cb(CombineArgs a, cudaStream_t st) {
    auto kern = combine_kernel<W, F32, SH, RS, RNR>;
    a.chunk = combine_chunk<W>(a.K, a.row_bytes);
    a.nchunks = (a.row_bytes + a.chunk - 1) / a.chunk;
    const size_t smem = combine_smem(a.K, a.chunk);
    static KernelSlots<decltype(kern)> slots;
    int sms = 0, per_sm = 0;
    cudaError_t e = slots.prepare(kern, CbShape<W>::THREADS, smem, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    const long long nitems = (long long)a.S * a.nchunks;
    long long grid = (long long)sms * per_sm;
    if (grid > nitems) grid = nitems;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(CbShape<W>::THREADS), smem, st, a);
}

template <int W, bool F32>
static cudaError_t launch_cb_dt(const CombineArgs &a, cudaStream_t st) {
    const bool sh = a.shared_out, rs = a.residual, rnr = a.out_no_routed;
    if (sh && rs && rnr) return launch_cb<W, F32, true, true, true>(a, st);
    if (sh && rs) return launch_cb<W, F32, true, true, false>(a, st);
    if (sh) return launch_cb<W, F32, true, false, false>(a, st);
    if (rs) return launch_cb<W, F32, false, true, false>(a, st);
    return launch_cb<W, F32, false, false, false>(a, st);
}

cudaError_t launch_combine(const void *y, int dtype, int S, int H, int K, int64_t cap,
                           const int32_t *slot_of, const float *topk_w, const void *shared_out,
                           const void *residual, void *out, void *out_no_routed, int32_t *status,
                           cudaStream_t st) {
    if (S == 0) return cudaSuccess;
    const bool f32 = dtype == MOE_DTYPE_F32;
    CombineArgs a;
    a.y = reinterpret_cast<const uint8_t *>(y);
    a.slot_of = slot_of;
    a.topk_w = topk_w;
    a.shared_out = reinterpret_cast<const uint8_t *>(shared_out);
    a.residual = reinterpret_cast<const uint8_t *>(residual);
    a.out = reinterpret_cast<uint8_t *>(out);
    a.out_no_routed = reinterpret_cast<uint8_t *>(out_no_routed);
    a.status = status;
    a.cap = cap;
    a.S = S;
    a.K = K;
    a.row_bytes = H * (f32 ? 4 : 2);
    if (a.row_bytes > 2048 && a.row_bytes <= 8192)
        return f32 ? launch_cb_dt<CB_MID_WARPS, true>(a, st) : launch_cb_dt<CB_MID_WARPS, false>(a, st);
    return f32 ? launch_cb_dt<8, true>(a, st) : launch_cb_dt<8, false>(a, st);
}

}  // namespace moe
