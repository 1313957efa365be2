// Router top-K gating: one warp per logits row (the per-row routine is in
// route_core.cuh, shared with the fused route + dispatch kernel).
//
// "Efficient and portable mixture-of-experts communication", Introduction:
// each token is sent to the K experts with the highest router scores, and the
// expert outputs are added with weights from the router's distribution.
#include "common.cuh"
#include "kernels.cuh"
#include "route_core.cuh"

namespace moe {

template <int NPER>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int S,
                                                         int E, int K, int32_t *__restrict__ topk_idx,
                                                         float *__restrict__ topk_w) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < S; t += warps) {
        uint32_t key[NPER];
        load_route_keys<NPER>(logits + (size_t)t * E, E, lane, key);
        int my_e;
        float my_w;
        topk_softmax<NPER>(key, K, lane, my_e, my_w);
        if (lane < K) {
            topk_idx[(size_t)t * K + lane] = my_e;
            topk_w[(size_t)t * K + lane] = my_w;
        }
    }
}

// Warps (tokens in flight) per CTA: 4 spreads the 4096 prefill tokens over the
// SMs more evenly than 8 (4.38 against 4.72 us per call).
constexpr int RT_WARPS = 4;
template <int NPER>
static cudaError_t launch_route(const float *logits, int S, int E, int K, int32_t *idx, float *w,
                                cudaStream_t st, int sms) {
    const int threads = 32 * RT_WARPS;
    int blocks = (S + RT_WARPS - 1) / RT_WARPS;
    const int cap_blocks = sms * 64 / RT_WARPS;
    if (blocks > cap_blocks) blocks = cap_blocks;
    if (blocks < 1) blocks = 1;
    static KernelSlots<decltype(&route_topk_kernel<NPER>)> slots;
    int n_sms = 0, per_sm = 0;
    const cudaError_t e = slots.prepare(&route_topk_kernel<NPER>, threads, 0, &n_sms, &per_sm);
    if (e != cudaSuccess) return e;
    return launch_pdl(route_topk_kernel<NPER>, dim3(blocks), dim3(threads), 0, st, logits, S, E, K, idx, w);
}

cudaError_t launch_route_topk(const float *logits, int S, int E, int K, int32_t *idx, float *w,
                              cudaStream_t st, int sms) {
    const int nper = (E + 31) / 32;
    if (nper <= 1) return launch_route<1>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 2) return launch_route<2>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 4) return launch_route<4>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 8) return launch_route<8>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 12) return launch_route<12>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 16) return launch_route<16>(logits, S, E, K, idx, w, st, sms);
    if (nper <= 24) return launch_route<24>(logits, S, E, K, idx, w, st, sms);
    return launch_route<32>(logits, S, E, K, idx, w, st, sms);
}

// ------------------------------------------------------------------------------------------
// Router variant: sigmoid scores, selection-only bias, group-limited top-K (the
// DeepSeek-V3 router that "Efficient and portable mixture-of-experts
// communication" cites; plainest reading).  exp is built from IEEE basic
// operations -- Cody-Waite reduction with a 16-bit head of ln 2, the degree-7
// Taylor polynomial in Horner form, two exact power-of-two factors -- and every
// operation below is an explicit round-to-nearest intrinsic (no contraction), so
// the selection scores are the same fp32 values the oracle computes.
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

__device__ __forceinline__ float route_exp(float x) {
    if (x > 88.72283935546875f) return __int_as_float(0x7f800000);
    if (x < -103.97208404541015625f) return 0.0f;
    const float n = rintf(__fmul_rn(x, 1.44269502162933349609375f));
    float r = __fmaf_rn(-n, 0.693145751953125f, x);
    r = __fmaf_rn(-n, 1.428606765330187045037746429443359375e-06f, r);
    float p = 1.9841270114e-04f;
    p = __fmaf_rn(p, r, 1.3888889225e-03f);
    p = __fmaf_rn(p, r, 8.3333337680e-03f);
    p = __fmaf_rn(p, r, 4.1666667908e-02f);
    p = __fmaf_rn(p, r, 1.6666667163e-01f);
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int ni = (int)n;
    const int h = ni / 2;
    return __fmul_rn(__fmul_rn(p, pow2i(h)), pow2i(ni - h));
}

__device__ __forceinline__ float route_sigmoid(float l) {
    return __fdiv_rn(1.0f, __fadd_rn(1.0f, route_exp(-l)));
}

// One warp per token; lane holds experts e = lane + 32 j (j < NPER).  The
// warp also keeps the row's scores in its own shared-memory slice, [E]
// selection scores then [E] sigmoid scores, so that (1) the group scores are
// scanned by LPG lanes per group (LPG = 32 / n_group rounded down to a power
// of two) followed by an xor merge of (largest, second largest), and (2) the
// winner's sigmoid score is one broadcast shared load.
constexpr int SG_WARPS = 8;

template <int NPER>
__global__ void __launch_bounds__(SG_WARPS * 32)
    route_sigmoid_grouped_kernel(const float *__restrict__ logits, const float *__restrict__ bias, int S, int E,
                                 int K, int n_group, int topk_group, int normalize, float scale,
                                 int32_t *__restrict__ topk_idx, float *__restrict__ topk_w) {
    extern __shared__ float sg_smem[];
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    float *const cs = sg_smem + (size_t)wib * 2 * E;  // selection scores of the warp's row
    float *const ss = cs + E;                         // sigmoid scores
    const int warps = (gridDim.x * blockDim.x) >> 5;
    const int gsize = E / n_group;
    int lpg = 1;  // lanes per group
    while (lpg * 2 * n_group <= 32) lpg *= 2;
    const int my_g = lane / lpg, my_sub = lane - my_g * lpg;
    const float NEG_INF = __int_as_float(0xff800000);
    // group of expert e (< 1024) = umulhi(e, ceil(2^32 / gsize)), exact for gsize >= 2
    const uint32_t gmagic = n_group > 1 ? 0xffffffffu / (uint32_t)gsize + 1u : 0u;
    float bv[NPER];
#pragma unroll
    for (int j = 0; j < NPER; ++j) bv[j] = (bias && lane + 32 * j < E) ? __ldg(bias + lane + 32 * j) : 0.f;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < S; t += warps) {
        const float *row = logits + (size_t)t * E;
        float lv[NPER];
#pragma unroll
        for (int j = 0; j < NPER; ++j) lv[j] = lane + 32 * j < E ? __ldg(row + lane + 32 * j) : 0.f;
        float cv[NPER];
#pragma unroll
        for (int j = 0; j < NPER; ++j) {
            const int e = lane + 32 * j;
            cv[j] = NEG_INF;  // not an expert
            if (e < E) {
                // sigmoid = 1 / (1 + exp(-l)): the correctly rounded reciprocal is the
                // correctly rounded quotient 1 / d
                const float sg = __frcp_rn(__fadd_rn(1.0f, route_exp(-lv[j])));
                cv[j] = bias ? __fadd_rn(sg, bv[j]) : sg;
                cs[e] = cv[j];
                ss[e] = sg;
            }
        }
        __syncwarp();
        // ---- groups: score = largest + second largest selection score ----
        uint32_t keep = 0xffffffffu;  // bit (g * lpg) set: group g kept
        if (n_group > 1) {
            float a1 = NEG_INF, a2 = NEG_INF;
            if (my_g < n_group) {
                // each group starts its scan at a different offset, so the lanes of
                // one step read distinct banks (order does not change a top-2)
                const float *grp = cs + my_g * gsize;
                const int shift = (my_g * lpg) % gsize;
                for (int i = my_sub; i < gsize; i += lpg) {
                    const int j = i + shift < gsize ? i + shift : i + shift - gsize;
                    const float v = grp[j];
                    a2 = fmaxf(a2, fminf(a1, v));
                    a1 = fmaxf(a1, v);
                }
            }
            for (int m = 1; m < lpg; m <<= 1) {
                const float b1 = __shfl_xor_sync(FULL, a1, m), b2 = __shfl_xor_sync(FULL, a2, m);
                const float n2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
                a1 = fmaxf(a1, b1);
                a2 = n2;
            }
            const bool leader = my_g < n_group && my_sub == 0;
            const uint32_t gkey = leader ? ordered_bits(__fadd_rn(a1, a2)) : 0u;
            bool taken = false;
            // keep the topk_group best groups (ties: lower group = lower lane)
            for (int r = 0; r < topk_group; ++r) {
                const uint32_t key = (leader && !taken) ? gkey : 0u;
                const uint32_t best = __reduce_max_sync(FULL, key);
                const uint32_t win =
                    __reduce_min_sync(FULL, (leader && !taken && gkey == best) ? (uint32_t)lane : 0xffffffffu);
                if ((uint32_t)lane == win) taken = true;
            }
            keep = __ballot_sync(FULL, taken);
        }
        // ---- top-K of the selection score over the experts of the kept groups ----
        uint32_t key[NPER];
#pragma unroll
        for (int j = 0; j < NPER; ++j) {
            const int e = lane + 32 * j;
            bool ok = e < E;
            if (n_group > 1 && ok) ok = (keep >> (__umulhi((uint32_t)e, gmagic) * lpg)) & 1u;
            key[j] = ok ? ordered_bits(cv[j]) : 0u;
        }
        int my_e = 0;
        for (int k = 0; k < K; ++k) {
            uint32_t m = key[0];
#pragma unroll
            for (int j = 1; j < NPER; ++j) m = max(m, key[j]);
            const uint32_t best = __reduce_max_sync(FULL, m);
            uint32_t cand = 0xffffffffu;
#pragma unroll
            for (int j = NPER - 1; j >= 0; --j) cand = key[j] == best ? (uint32_t)(lane + 32 * j) : cand;
            const uint32_t win = __reduce_min_sync(FULL, cand);
            if (lane == k) my_e = (int)win;
#pragma unroll
            for (int j = 0; j < NPER; ++j) key[j] = (uint32_t)(lane + 32 * j) == win ? 0u : key[j];
        }
        // the winners' unbiased scores (an id past E only from NaN logits: read as 0)
        const float my_s = (lane < K && (unsigned)my_e < (unsigned)E) ? ss[my_e] : 0.f;
        float sum = 0.f;  // in k order, as the oracle
        for (int k = 0; k < K; ++k) sum = __fadd_rn(sum, __shfl_sync(FULL, my_s, k));
        if (lane < K) {
            const float v = normalize ? __fdiv_rn(my_s, sum) : my_s;
            topk_idx[(size_t)t * K + lane] = my_e;
            topk_w[(size_t)t * K + lane] = __fmul_rn(v, scale);
        }
        __syncwarp();  // the slice is rewritten by the warp's next token
    }
}

template <int NPER>
static cudaError_t launch_sg(const float *logits, const float *bias, int S, int E, int K, int n_group,
                             int topk_group, int normalize, float scale, int32_t *idx, float *w, cudaStream_t st,
                             int sms) {
    const int threads = SG_WARPS * 32;
    const size_t smem = (size_t)SG_WARPS * 2 * E * sizeof(float);
    static KernelSlots<decltype(&route_sigmoid_grouped_kernel<NPER>)> slots;
    int n_sms = 0, per_sm = 0;
    const cudaError_t e = slots.prepare(&route_sigmoid_grouped_kernel<NPER>, threads, smem, &n_sms, &per_sm);
    if (e != cudaSuccess) return e;
    long long blocks = ((long long)S + SG_WARPS - 1) / SG_WARPS;
    const long long resident = (long long)n_sms * (per_sm > 0 ? per_sm : 1);
    if (blocks > resident) blocks = resident;
    if (blocks < 1) blocks = 1;
    return launch_pdl(route_sigmoid_grouped_kernel<NPER>, dim3((unsigned)blocks), dim3(threads), smem, st, logits,
                      bias, S, E, K, n_group, topk_group, normalize, scale, idx, w);
}

cudaError_t launch_route_sigmoid_grouped(const float *logits, const float *bias, int S, int E, int K, int n_group,
                                         int topk_group, int normalize, float scale, int32_t *idx, float *w,
                                         cudaStream_t st, int sms) {
    const int nper = (E + 31) / 32;
#define MOE_SG(N) return launch_sg<N>(logits, bias, S, E, K, n_group, topk_group, normalize, scale, idx, w, st, sms)
    if (nper <= 1) MOE_SG(1);
    if (nper <= 2) MOE_SG(2);
    if (nper <= 4) MOE_SG(4);
    if (nper <= 8) MOE_SG(8);
    if (nper <= 12) MOE_SG(12);
    if (nper <= 16) MOE_SG(16);
    if (nper <= 24) MOE_SG(24);
    MOE_SG(32);
#undef MOE_SG
}

// Backward through the gating softmax: for the selected experts
// grad_logits[t, e_k] = w_k (gw_k - sum_j w_j gw_j), 0 for the others.  One warp
// per token: the dense row is zeroed, then lanes k < K write their entries
// (ids outside [0, E) are skipped).
__global__ void __launch_bounds__(256) route_backward_kernel(const int32_t *__restrict__ topk_idx,
                                                             const float *__restrict__ topk_w,
                                                             const float *__restrict__ grad_w, int S, int E,
                                                             int K, float *__restrict__ grad_logits) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < S; t += warps) {
        float w = 0.f, gw = 0.f;
        int e = -1;
        if (lane < K) {
            w = __ldg(topk_w + (size_t)t * K + lane);
            gw = __ldg(grad_w + (size_t)t * K + lane);
            e = __ldg(topk_idx + (size_t)t * K + lane);
        }
        float dot = __fmul_rn(w, gw);
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) dot += __shfl_xor_sync(FULL, dot, m);
        float *row = grad_logits + (size_t)t * E;
        for (int j = lane; j < E; j += 32) row[j] = 0.f;
        __syncwarp();
        if (lane < K && e >= 0 && e < E) row[e] = __fmul_rn(w, __fsub_rn(gw, dot));
    }
}

cudaError_t launch_route_backward(const int32_t *topk_idx, const float *topk_w, const float *grad_w, int S,
                                  int E, int K, float *grad_logits, cudaStream_t st, int sms) {
    const int threads = 256;
    int blocks = (S + 7) / 8;
    if (blocks > sms * 8) blocks = sms * 8;
    if (blocks < 1) blocks = 1;
    static KernelSlots<decltype(&route_backward_kernel)> slots;
    int n_sms = 0, per_sm = 0;
    const cudaError_t e = slots.prepare(&route_backward_kernel, threads, 0, &n_sms, &per_sm);
    if (e != cudaSuccess) return e;
    return launch_pdl(route_backward_kernel, dim3(blocks), dim3(threads), 0, st, topk_idx, topk_w, grad_w, S, E,
                      K, grad_logits);
}

}  // namespace moe
