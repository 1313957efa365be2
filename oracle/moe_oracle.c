/*
 * CPU oracle for MoE token dispatch and combine — TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
 * leg may load or call this file.  The product path (the CUDA library under
 * combine_moe_route_09_b200/) never does, and this file shares no code, header,
 * table or helper with it.
 *
 * Every function is the plain definition of one step, written with loops in
 * the order the pages state it, single-threaded, with no blocking or fusion:
 *
 *   oracle_route_topk   router top-K selection and gating weights
 *   oracle_layout       per-expert counts, padded offsets, slot assignment
 *   oracle_dispatch     scatter of token rows (optionally FP8 e4m3, 128-ch blocks)
 *   oracle_combine      gather + top-K weighted sum + dual-residual epilogue
 *   oracle_combine_fp8  the combine over e4m3 expert outputs with block scales
 *   oracle_route_sigmoid_grouped   router variant: sigmoid scores, selection-only
 *                       bias, group-limited top-K (with its exp / sigmoid)
 *   oracle_route_weights_dispatched   routing weights in dispatched row order
 *   oracle_combine_backward / oracle_dispatch_backward / oracle_route_backward
 *                       the transposes of the steps (training)
 *   oracle_e4m3_encode / oracle_e4m3_decode / oracle_bf16_round   format helpers
 *
 * Sources (page title, section):
 *   [pplx]    "Efficient and portable mixture-of-experts communication"
 *             (Perplexity blog on pplx-kernels): Introduction; Portable Kernels;
 *             Dispatch; Combine.
 *   [farskip] Instella-MoE-16B-A3B-SFT / FarSkip-Collective explainer
 *             (hotelren.com news 5835394): "the dual residual stream" and the
 *             four-line update in "where the dual residual is implemented".
 *   [deepep]  "DeepSeek AI releases DeepEP": Technical overview (FP8 dispatch).
 *   [moonep]  "MoonEP developer guide": core API example (tokens_per_expert,
 *             cu_seqlens, plan) and performance tuning (token_padding, 128).
 *
 * Precision: the workloads fix fp32 router logits, bf16 or fp32 activations,
 * fp32 FP8 scales and an fp32 combine accumulator; the oracle computes those
 * steps in exactly that precision.  The gating softmax is computed in fp64 and
 * rounded once to fp32.  Compile with -O2 -ffp-contract=off (no fast-math) so
 * that every float operation is the single IEEE operation written here.
 *
 * Parity status of each function is recorded in the pin tests
 * (tests/test_oracle_*.py); every function here is pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_EINDEX 2
#define ORACLE_EOVERFLOW 3

#define ORACLE_DTYPE_F32 0
#define ORACLE_DTYPE_BF16 1
#define ORACLE_QUANT_NONE 0
#define ORACLE_QUANT_FP8_E4M3_B128 1

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper half of an fp32 bit pattern, so widening is exact. */
static float bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/*
 * fp32 -> bf16, round to nearest, ties to the even bf16 pattern.  Written from
 * the definition: the two bf16 neighbours of v are the truncated pattern and
 * the next one up in magnitude, one bf16 step (2^(exponent-7)) further out;
 * pick the nearer (compared exactly in fp64), and on a tie the one whose last
 * bit is 0.  Past the largest finite bf16 the next pattern is infinity, valued
 * 2^128 for the comparison, as round-to-nearest overflow requires.
 */
uint16_t oracle_bf16_round(float v)
{
    uint32_t u = f32_to_bits(v);
    if (isnan(v)) return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    if (isinf(v)) return (uint16_t)(u >> 16);
    uint16_t lo = (uint16_t)(u >> 16);            /* toward zero */
    uint16_t hi = (uint16_t)(lo + 1);             /* away from zero (may become inf) */
    int ebits = (lo >> 7) & 0xFF;
    double step = ldexp(1.0, (ebits == 0 ? 1 : ebits) - 127 - 7);
    double a = fabs((double)v);
    double vlo = fabs((double)bf16_to_f32(lo));
    double vhi = vlo + step;
    double dlo = a - vlo, dhi = vhi - a;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo & 1u) ? hi : lo;
}

/*
 * FP8 e4m3 ("fn" variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits; no infinities; 0x7F / 0xFF are NaN; largest finite magnitude 448
 * (code 0x7E).  Exponent field 0 holds the subnormals m * 2^-9, m = 1..7.
 */
float oracle_e4m3_decode(uint8_t q)
{
    int sign = q >> 7, ex = (q >> 3) & 0xF, m = q & 7;
    double mag;
    if (ex == 0xF && m == 7) return NAN;
    if (ex == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, ex - 7);
    return (float)(sign ? -mag : mag);
}

/*
 * fp32 -> e4m3, round to nearest with ties to the even code, saturating to
 * +-448 (the FP8 dispatch never produces NaN from finite input).  Written from
 * the definition: the non-negative finite codes 0x00..0x7E are increasing in
 * value, so find by bisection the pair of adjacent codes around |v|, take the
 * nearer, and on a tie the even code.  The sign bit is copied (so -0.0 -> 0x80).
 */
uint8_t oracle_e4m3_encode(float v)
{
    uint8_t sign = (f32_to_bits(v) >> 31) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (isnan(v)) return 0x7F;
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 0x7E; /* invariant: value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if ((double)oracle_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    double dlo = a - (double)oracle_e4m3_decode((uint8_t)lo);
    double dhi = (double)oracle_e4m3_decode((uint8_t)hi) - a;
    int code;
    if (dlo < dhi) code = lo;
    else if (dhi < dlo) code = hi;
    else code = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)(sign | code);
}

/* ------------------------------------------------------------------------ */
/* Step 1: router top-K gating                                                */
/* ------------------------------------------------------------------------ */

/*
 * [pplx] Introduction: each token goes to the K experts with the highest router
 * scores, and the layer output adds the expert outputs times a weight taken
 * from the router's probability distribution.
 *
 * Selection: K passes, each taking the largest logit not yet chosen; a strict
 * ">" makes the lower expert id win a tie, and -0.0 == +0.0 as C compares
 * them.  Output is in selection order (descending logit, ascending id on ties).
 *
 * Weights: softmax over the K selected logits,
 *     w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0),   l_0 the largest,
 * which equals the full softmax over all E experts renormalised over the
 * chosen K.  Evaluated in fp64, rounded once to fp32.
 * Precondition: finite logits, 1 <= K <= E.
 */
int oracle_route_topk(const float *logits, int S, int E, int K,
                      int32_t *topk_idx, float *topk_w)
{
    if (S < 0 || E < 1 || K < 1 || K > E) return ORACLE_EINVAL;
    char *taken = (char *)malloc((size_t)E);
    double *ex = (double *)malloc(sizeof(double) * (size_t)K);
    if (!taken || !ex) { free(taken); free(ex); return ORACLE_EINVAL; }
    for (int t = 0; t < S; ++t) {
        const float *row = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || row[e] > row[best]) best = e;
            }
            taken[best] = 1;
            topk_idx[(size_t)t * K + k] = best;
        }
        double l0 = (double)row[topk_idx[(size_t)t * K]];
        double sum = 0.0;
        for (int k = 0; k < K; ++k) {
            ex[k] = exp((double)row[topk_idx[(size_t)t * K + k]] - l0);
            sum += ex[k];
        }
        for (int k = 0; k < K; ++k) topk_w[(size_t)t * K + k] = (float)(ex[k] / sum);
    }
    free(taken);
    free(ex);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Step 2: per-expert histogram and prefix scan into the dispatched layout    */
/* ------------------------------------------------------------------------ */

/*
 * [moonep] core API example: dispatch returns tokens_per_expert and cu_seqlens
 * (the running start of each expert's rows); performance tuning: each expert
 * group is padded to token_padding rows (default 128).
 * [pplx] Portable Kernels: each (source rank, local expert) receive region has
 * a fixed upper bound, so every write address is known without sync; experts
 * are split over ranks in blocks of num_experts // EP.
 * [pplx] Dispatch: the receiver keeps, per routed token, the source rank,
 * expert index and token index for the combine, and packs tokens of one expert
 * contiguously regardless of sender; the arrival order there is not fixed.
 *
 * Definitions (pairs i = t*K + k in ascending order):
 *   counts[e]      = #{ i : topk_idx[i] == e }
 *   pc[e]          = P > 0 ? ceil(counts[e] / P) * P : counts[e]
 *   offsets[0]     = 0,  offsets[e+1] = offsets[e] + pc[e]
 *   rank_offsets[r]= offsets[r * (E/R)],  r = 0..R
 *   slot_of[i]     = offsets[e] + #{ i' < i : topk_idx[i'] == e }   (stable)
 *   row_src[s]     = i if slot_of[i] == s, else -1   (s < cap)
 * The stable (ascending pair index) order fixes the order the pages leave free;
 * because experts of one rank are a contiguous id block, the layout is
 * rank-major, then local expert, then slot.
 * Errors: an index outside [0,E) -> ORACLE_EINDEX; offsets[E] > cap ->
 * ORACLE_EOVERFLOW.  Outputs are only complete when ORACLE_OK is returned.
 */
int oracle_layout(const int32_t *topk_idx, int S, int E, int K, int R, int P,
                  int64_t cap, int32_t *counts, int32_t *offsets,
                  int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src)
{
    if (S < 0 || E < 1 || K < 1 || R < 1 || E % R != 0 || P < 0 || cap < 0)
        return ORACLE_EINVAL;
    int64_t npairs = (int64_t)S * K;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < npairs; ++i) {
        int32_t e = topk_idx[i];
        if (e < 0 || e >= E) return ORACLE_EINDEX;
        counts[e] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int64_t pc = counts[e];
        if (P > 0) pc = ((pc + P - 1) / P) * P;
        offsets[e + 1] = (int32_t)(offsets[e] + pc);
    }
    int Eloc = E / R;
    for (int r = 0; r <= R; ++r) rank_offsets[r] = offsets[r * Eloc];
    if ((int64_t)offsets[E] > cap) return ORACLE_EOVERFLOW;
    for (int64_t s = 0; s < cap; ++s) row_src[s] = -1;
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!fill) return ORACLE_EINVAL;
    for (int64_t i = 0; i < npairs; ++i) {
        int32_t e = topk_idx[i];
        int32_t s = offsets[e] + fill[e];
        fill[e] += 1;
        slot_of[i] = s;
        row_src[s] = (int32_t)i;
    }
    free(fill);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Step 3: dispatch (scatter), optionally FP8 e4m3 per 128-channel block      */
/* ------------------------------------------------------------------------ */

/*
 * [pplx] Dispatch: the sender packs each routed token's activations (with its
 * block scaling factors when quantised) and the receiver lays them out
 * contiguously per expert for the grouped GEMM.  [deepep] Technical overview:
 * the dispatch may carry FP8.  Scale rule (the workloads' statement): one fp32
 * scale per 128-channel block, s = amax / 448, codes round to nearest even.
 *
 *   no quantisation:  xd[slot_of[t,k], :] = x[t, :]   (same dtype, bit copy)
 *   FP8:  for block j of row t (channels 128j .. 128j+127):
 *           amax = max |x[t,c]|  (bf16 widened exactly to fp32)
 *           s    = amax / 448                      (fp32 division)
 *           q[c] = e4m3_rn_sat(x[t,c] / s)         (fp32 division, then RNE)
 *           if s == 0 every q is a signed zero (0x00, or 0x80 for -0.0)
 *         xd[slot, c] = q[c] (uint8), xs[slot, j] = s, for every k.
 * Rows of xd that no pair maps to (padding) are not written.  Pairs whose
 * slot_of is negative are skipped.  A slot >= cap -> ORACLE_EOVERFLOW.
 */
int oracle_dispatch(const void *x, int dtype, int S, int H, int K,
                    const int32_t *slot_of, int quant, int64_t cap,
                    void *xd, float *xs)
{
    if (S < 0 || H < 1 || K < 1) return ORACLE_EINVAL;
    if (dtype != ORACLE_DTYPE_F32 && dtype != ORACLE_DTYPE_BF16) return ORACLE_EINVAL;
    if (quant != ORACLE_QUANT_NONE && quant != ORACLE_QUANT_FP8_E4M3_B128) return ORACLE_EINVAL;
    if (quant == ORACLE_QUANT_FP8_E4M3_B128 && (H % 128 != 0 || !xs)) return ORACLE_EINVAL;
    size_t esz = dtype == ORACLE_DTYPE_F32 ? 4 : 2;
    int nb = H / 128;
    float *row = (float *)malloc(sizeof(float) * (size_t)H);
    uint8_t *q = (uint8_t *)malloc((size_t)H);
    float *sc = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    if (!row || !q || !sc) { free(row); free(q); free(sc); return ORACLE_EINVAL; }
    int rc = ORACLE_OK;
    for (int t = 0; t < S; ++t) {
        if (quant == ORACLE_QUANT_FP8_E4M3_B128) {
            for (int c = 0; c < H; ++c)
                row[c] = dtype == ORACLE_DTYPE_F32
                             ? ((const float *)x)[(size_t)t * H + c]
                             : bf16_to_f32(((const uint16_t *)x)[(size_t)t * H + c]);
            for (int j = 0; j < nb; ++j) {
                float amax = 0.0f;
                for (int c = 128 * j; c < 128 * j + 128; ++c)
                    if (fabsf(row[c]) > amax) amax = fabsf(row[c]);
                float s = amax / 448.0f;
                sc[j] = s;
                for (int c = 128 * j; c < 128 * j + 128; ++c) {
                    if (s == 0.0f) q[c] = (f32_to_bits(row[c]) >> 31) ? 0x80 : 0x00;
                    else q[c] = oracle_e4m3_encode(row[c] / s);
                }
            }
        }
        for (int k = 0; k < K; ++k) {
            int32_t s = slot_of[(size_t)t * K + k];
            if (s < 0) continue;
            if ((int64_t)s >= cap) { rc = ORACLE_EOVERFLOW; continue; }
            if (quant == ORACLE_QUANT_FP8_E4M3_B128) {
                memcpy((uint8_t *)xd + (size_t)s * H, q, (size_t)H);
                memcpy(xs + (size_t)s * nb, sc, sizeof(float) * (size_t)nb);
            } else {
                memcpy((uint8_t *)xd + (size_t)s * H * esz,
                       (const uint8_t *)x + (size_t)t * H * esz, (size_t)H * esz);
            }
        }
    }
    free(row); free(q); free(sc);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Step 4: combine (gather + top-K weighted sum) with the dual residual       */
/* ------------------------------------------------------------------------ */

/*
 * [pplx] Combine: the receiver reads each token's expert outputs from the
 * buffers the routing table names and forms their router-weighted sum.
 * [farskip] the dual residual stream: the MoE block returns the full output
 * (routed + shared) and the shared-only output; then
 *     residual_no_routed = residual + shared_out
 *     residual           = residual + mlp_output,  mlp_output = shared_out + routed
 *
 * Per token t and channel h, in fp32 (the workloads' fp32 accumulate), in
 * exactly this order:
 *     acc = 0; for k = 0..K-1 (slot_of >= 0): acc = fma(w[t,k], y[slot,h], acc)
 *     m   = shared[t,h] + acc                 (if shared given, else m = acc)
 *     out = residual[t,h] + m                 (if residual given, else out = m)
 *     rnr = residual[t,h] + shared[t,h]       (only when both are given)
 * Each output is rounded once to the I/O dtype (bf16: nearest-even).
 * out_no_routed must be NULL unless both shared and residual are given.
 * A slot >= cap -> ORACLE_EOVERFLOW (the pair is skipped).
 */
int oracle_combine(const void *y, int dtype, int S, int H, int K, int64_t cap,
                   const int32_t *slot_of, const float *topk_w,
                   const void *shared, const void *residual,
                   void *out, void *out_no_routed)
{
    if (S < 0 || H < 1 || K < 1) return ORACLE_EINVAL;
    if (dtype != ORACLE_DTYPE_F32 && dtype != ORACLE_DTYPE_BF16) return ORACLE_EINVAL;
    if (out_no_routed && !(shared && residual)) return ORACLE_EINVAL;
    int rc = ORACLE_OK;
    for (int t = 0; t < S; ++t) {
        for (int k = 0; k < K; ++k) {
            int32_t s = slot_of[(size_t)t * K + k];
            if (s >= 0 && (int64_t)s >= cap) rc = ORACLE_EOVERFLOW;
        }
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int32_t s = slot_of[(size_t)t * K + k];
                if (s < 0 || (int64_t)s >= cap) continue;
                size_t yi = (size_t)s * H + h;
                float yv = dtype == ORACLE_DTYPE_F32 ? ((const float *)y)[yi]
                                                     : bf16_to_f32(((const uint16_t *)y)[yi]);
                acc = fmaf(topk_w[(size_t)t * K + k], yv, acc);
            }
            size_t oi = (size_t)t * H + h;
            float sh = 0.0f, rs = 0.0f;
            if (shared)
                sh = dtype == ORACLE_DTYPE_F32 ? ((const float *)shared)[oi]
                                               : bf16_to_f32(((const uint16_t *)shared)[oi]);
            if (residual)
                rs = dtype == ORACLE_DTYPE_F32 ? ((const float *)residual)[oi]
                                               : bf16_to_f32(((const uint16_t *)residual)[oi]);
            float m = shared ? sh + acc : acc;
            float o = residual ? rs + m : m;
            if (dtype == ORACLE_DTYPE_F32) ((float *)out)[oi] = o;
            else ((uint16_t *)out)[oi] = oracle_bf16_round(o);
            if (out_no_routed) {
                float n = rs + sh;
                if (dtype == ORACLE_DTYPE_F32) ((float *)out_no_routed)[oi] = n;
                else ((uint16_t *)out_no_routed)[oi] = oracle_bf16_round(n);
            }
        }
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Backward of the path (training): the transposes of the steps above        */
/* ------------------------------------------------------------------------ */

/*
 * Backward of oracle_combine.  "MoonEP developer guide", core API example:
 * the backward pass reuses the plan (dispatch of grad_output, combine of the
 * expert gradients).  With g = dL/d(residual_out) and gn = dL/d(residual_no_routed)
 * (zero if not given), the forward out = residual + (shared + sum_k w_k y_k),
 * rnr = residual + shared gives, per token t and pair k with a valid slot:
 *     grad_y[slot, h]  = w[t,k] * g[t,h]          (fp32 product, rounded once)
 *     grad_w[t, k]     = sum_h y[slot, h] * g[t,h] (fp64, rounded once to fp32)
 *     grad_skip[t, h]  = g[t,h] + gn[t,h]         (fp32, rounded once) -- the
 *                        gradient of both `residual` and `shared_out`
 * grad_w is 0 for skipped pairs; rows of grad_y no pair maps to are untouched.
 */
int oracle_combine_backward(const void *g, const void *gn, const void *y, int dtype, int S, int H,
                            int K, int64_t cap, const int32_t *slot_of, const float *topk_w,
                            void *grad_y, float *grad_w, void *grad_skip)
{
    if (S < 0 || H < 1 || K < 1) return ORACLE_EINVAL;
    if (dtype != ORACLE_DTYPE_F32 && dtype != ORACLE_DTYPE_BF16) return ORACLE_EINVAL;
    int f32 = dtype == ORACLE_DTYPE_F32;
#define LD(p, i) (f32 ? ((const float *)(p))[i] : bf16_to_f32(((const uint16_t *)(p))[i]))
    for (int t = 0; t < S; ++t) {
        for (int k = 0; k < K; ++k) {
            int32_t s = slot_of[(size_t)t * K + k];
            double dot = 0.0;
            if (s >= 0 && (int64_t)s < cap) {
                float w = topk_w[(size_t)t * K + k];
                for (int h = 0; h < H; ++h) {
                    float gv = LD(g, (size_t)t * H + h);
                    float prod = w * gv;
                    if (f32) ((float *)grad_y)[(size_t)s * H + h] = prod;
                    else ((uint16_t *)grad_y)[(size_t)s * H + h] = oracle_bf16_round(prod);
                    dot += (double)LD(y, (size_t)s * H + h) * (double)gv;
                }
            }
            grad_w[(size_t)t * K + k] = (float)dot;
        }
        if (grad_skip) {
            for (int h = 0; h < H; ++h) {
                size_t i = (size_t)t * H + h;
                float v = gn ? LD(g, i) + LD(gn, i) : LD(g, i);
                if (f32) ((float *)grad_skip)[i] = v;
                else ((uint16_t *)grad_skip)[i] = oracle_bf16_round(v);
            }
        }
    }
#undef LD
    return ORACLE_OK;
}

/*
 * Backward of oracle_dispatch (the plain copy; for the FP8 dispatch the
 * quantiser is passed straight through): every copy of token t received x[t],
 * so grad_x[t, h] = sum over k with a valid slot of grad_xd[slot, h], summed in
 * fp32 in ascending k and rounded once (zero when no copy is valid).
 */
int oracle_dispatch_backward(const void *grad_xd, int dtype, int S, int H, int K, int64_t cap,
                             const int32_t *slot_of, void *grad_x)
{
    if (S < 0 || H < 1 || K < 1) return ORACLE_EINVAL;
    if (dtype != ORACLE_DTYPE_F32 && dtype != ORACLE_DTYPE_BF16) return ORACLE_EINVAL;
    int f32 = dtype == ORACLE_DTYPE_F32;
    for (int t = 0; t < S; ++t) {
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int32_t s = slot_of[(size_t)t * K + k];
                if (s < 0 || (int64_t)s >= cap) continue;
                size_t i = (size_t)s * H + h;
                acc += f32 ? ((const float *)grad_xd)[i] : bf16_to_f32(((const uint16_t *)grad_xd)[i]);
            }
            size_t o = (size_t)t * H + h;
            if (f32) ((float *)grad_x)[o] = acc;
            else ((uint16_t *)grad_x)[o] = oracle_bf16_round(acc);
        }
    }
    return ORACLE_OK;
}

/*
 * Route weights in dispatched order (MoonEP developer guide, core API example:
 * the dispatch also returns the routing weights of the rows it sends, which the
 * combine consumes).  Row slot_of[t,k] of the dispatched buffer carries
 * topk_w[t,k]; every other row of [0, cap) -- padding, unused capacity, pairs
 * dropped for a bad slot -- carries 0.
 */
int oracle_route_weights_dispatched(const float *topk_w, const int32_t *slot_of, int S, int K, int64_t cap,
                                    float *route_weights)
{
    if (S < 0 || K < 1 || cap < 0) return ORACLE_EINVAL;
    for (int64_t r = 0; r < cap; ++r) route_weights[r] = 0.0f;
    for (int t = 0; t < S; ++t)
        for (int k = 0; k < K; ++k) {
            int32_t s = slot_of[(size_t)t * K + k];
            if (s >= 0 && (int64_t)s < cap) route_weights[s] = topk_w[(size_t)t * K + k];
        }
    return ORACLE_OK;
}

/*
 * Backward of oracle_route_topk through the gating softmax.  The weights are
 * the softmax of the K selected logits, so for the selected experts
 *     grad_logits[t, e_k] = w_k * (gw_k - sum_j w_j gw_j)
 * and 0 for every expert not selected (the selection itself is piecewise
 * constant).  fp64, rounded once to fp32.
 */
int oracle_route_backward(const int32_t *topk_idx, const float *topk_w, const float *grad_w, int S,
                          int E, int K, float *grad_logits)
{
    if (S < 0 || E < 1 || K < 1 || K > E) return ORACLE_EINVAL;
    for (int t = 0; t < S; ++t) {
        double dotw = 0.0;
        for (int k = 0; k < K; ++k)
            dotw += (double)topk_w[(size_t)t * K + k] * (double)grad_w[(size_t)t * K + k];
        for (int e = 0; e < E; ++e) grad_logits[(size_t)t * E + e] = 0.0f;
        for (int k = 0; k < K; ++k) {
            int32_t e = topk_idx[(size_t)t * K + k];
            if (e < 0 || e >= E) return ORACLE_EINDEX;
            double w = topk_w[(size_t)t * K + k];
            grad_logits[(size_t)t * E + e] = (float)(w * ((double)grad_w[(size_t)t * K + k] - dotw));
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Combine over FP8 expert outputs                                            */
/* ------------------------------------------------------------------------ */

/*
 * oracle_combine with the expert outputs given as e4m3 codes plus one fp32
 * scale per 128-channel block (the format of the FP8 dispatch; "Efficient and
 * portable mixture-of-experts communication", Dispatch: tokens travel with
 * their block scaling factors).  Each element is dequantised as
 *     y = e4m3_value(q[slot, h]) * s[slot, h / 128]     (fp32 product)
 * and the accumulation and epilogue are those of oracle_combine; the
 * remaining arrays are in `dtype`.  H % 128 == 0.
 */
int oracle_combine_fp8(const uint8_t *yq, const float *ys, int dtype, int S, int H, int K, int64_t cap,
                       const int32_t *slot_of, const float *topk_w, const void *shared,
                       const void *residual, void *out, void *out_no_routed)
{
    if (S < 0 || H < 1 || K < 1 || H % 128 != 0) return ORACLE_EINVAL;
    if (dtype != ORACLE_DTYPE_F32 && dtype != ORACLE_DTYPE_BF16) return ORACLE_EINVAL;
    if (out_no_routed && !(shared && residual)) return ORACLE_EINVAL;
    int nb = H / 128, f32 = dtype == ORACLE_DTYPE_F32, rc = ORACLE_OK;
    for (int t = 0; t < S; ++t) {
        for (int k = 0; k < K; ++k) {
            int32_t s = slot_of[(size_t)t * K + k];
            if (s >= 0 && (int64_t)s >= cap) rc = ORACLE_EOVERFLOW;
        }
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int32_t s = slot_of[(size_t)t * K + k];
                if (s < 0 || (int64_t)s >= cap) continue;
                float yv = oracle_e4m3_decode(yq[(size_t)s * H + h]) * ys[(size_t)s * nb + h / 128];
                acc = fmaf(topk_w[(size_t)t * K + k], yv, acc);
            }
            size_t oi = (size_t)t * H + h;
            float sh = 0.0f, rs = 0.0f;
            if (shared) sh = f32 ? ((const float *)shared)[oi] : bf16_to_f32(((const uint16_t *)shared)[oi]);
            if (residual) rs = f32 ? ((const float *)residual)[oi] : bf16_to_f32(((const uint16_t *)residual)[oi]);
            float m = shared ? sh + acc : acc;
            float o = residual ? rs + m : m;
            if (f32) ((float *)out)[oi] = o;
            else ((uint16_t *)out)[oi] = oracle_bf16_round(o);
            if (out_no_routed) {
                float n = rs + sh;
                if (f32) ((float *)out_no_routed)[oi] = n;
                else ((uint16_t *)out_no_routed)[oi] = oracle_bf16_round(n);
            }
        }
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Router variant: sigmoid scores, selection-only bias, group-limited top-K   */
/* ------------------------------------------------------------------------ */

/*
 * exp(x) in fp32 from IEEE basic operations only, so that this oracle and the
 * CUDA kernel evaluate exactly the same sequence and take the same routing
 * decisions: Cody-Waite reduction x = n ln2 + r (n = RN(x log2 e), ln 2 split
 * into a 16-bit head, exact for |n| <= 256, and a tail), exp(r) by the degree-7
 * Taylor polynomial in Horner form with fma (|r| <= 0.35: truncation < 3e-9
 * relative), and 2^n applied as two exact power-of-two factors.  Pinned against
 * fp64 exp (within 2 ulp).  Below -104 the result is 0, above 88.72 it is inf.
 */
static float pow2i(int e) { return bits_to_f32((uint32_t)(e + 127) << 23); } /* -126 <= e <= 127 */

float oracle_route_exp(float x)
{
    if (x > 88.72283935546875f) return INFINITY;
    if (x < -103.97208404541015625f) return 0.0f;
    const float log2e = 1.44269502162933349609375f;       /* RN(1/ln 2) */
    const float ln2_hi = 0.693145751953125f;               /* ln 2 to 16 bits */
    const float ln2_lo = 1.428606765330187045037746429443359375e-06f; /* RN(ln 2 - ln2_hi) */
    float n = rintf(x * log2e);
    float r = fmaf(-n, ln2_hi, x);
    r = fmaf(-n, ln2_lo, r);
    float p = 1.9841270114e-04f;                /* 1/7! */
    p = fmaf(p, r, 1.3888889225e-03f);          /* 1/6! */
    p = fmaf(p, r, 8.3333337680e-03f);          /* 1/5! */
    p = fmaf(p, r, 4.1666667908e-02f);          /* 1/4! */
    p = fmaf(p, r, 1.6666667163e-01f);          /* 1/3! */
    p = fmaf(p, r, 0.5f);                       /* 1/2! */
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;
    int h = ni / 2;
    return (p * pow2i(h)) * pow2i(ni - h);
}

/* sigmoid(l) = 1 / (1 + exp(-l)), fp32, IEEE addition and division. */
float oracle_route_sigmoid(float l) { return 1.0f / (1.0f + oracle_route_exp(-l)); }

/*
 * Sigmoid routing with a selection-only bias and group-limited top-K (the
 * DeepSeek-V3 technical report, which "Efficient and portable
 * mixture-of-experts communication" cites for its router; the pages give no
 * detail, so this is the plainest reading):
 *   s_e = sigmoid(l_e)                          (the gating score)
 *   c_e = s_e + bias_e                          (the selection score; bias may be NULL)
 *   n_group > 1: the E experts form n_group contiguous groups; a group's score
 *     is (largest c) + (second largest c) in it (fp32, in that order); the
 *     topk_group highest groups (ties: lower group) stay, the rest are excluded
 *   top-K of c over the experts that stay (descending, ties: lower id)
 *   w_k = s_{e_k}; with normalize, w_k = s_{e_k} / (s_{e_0} + ... + s_{e_{K-1}})
 *     (sum in k order); then w_k = w_k * scale.   All fp32.
 * Requires E % n_group == 0, E / n_group >= 2, topk_group * E / n_group >= K.
 */
int oracle_route_sigmoid_grouped(const float *logits, const float *bias, int S, int E, int K, int n_group,
                                 int topk_group, int normalize, float scale, int32_t *topk_idx, float *topk_w)
{
    if (S < 0 || E < 1 || K < 1 || K > E || n_group < 1 || E % n_group != 0) return ORACLE_EINVAL;
    int gsize = E / n_group;
    if (n_group > 1 && (gsize < 2 || topk_group < 1 || topk_group > n_group || topk_group * gsize < K))
        return ORACLE_EINVAL;
    float *s = (float *)malloc(sizeof(float) * (size_t)E);
    float *c = (float *)malloc(sizeof(float) * (size_t)E);
    char *allowed = (char *)malloc((size_t)E);
    float *gs = (float *)malloc(sizeof(float) * (size_t)n_group);
    char *gtaken = (char *)malloc((size_t)n_group);
    if (!s || !c || !allowed || !gs || !gtaken) { free(s); free(c); free(allowed); free(gs); free(gtaken); return ORACLE_EINVAL; }
    for (int t = 0; t < S; ++t) {
        const float *row = logits + (size_t)t * E;
        for (int e = 0; e < E; ++e) {
            s[e] = oracle_route_sigmoid(row[e]);
            c[e] = bias ? s[e] + bias[e] : s[e];
            allowed[e] = 1;
        }
        if (n_group > 1) {
            for (int g = 0; g < n_group; ++g) {
                int b1 = -1, b2 = -1;
                for (int e = g * gsize; e < (g + 1) * gsize; ++e) {
                    if (b1 < 0 || c[e] > c[b1]) { b2 = b1; b1 = e; }
                    else if (b2 < 0 || c[e] > c[b2]) b2 = e;
                }
                gs[g] = c[b1] + c[b2];
                gtaken[g] = 0;
            }
            for (int r = 0; r < topk_group; ++r) {
                int best = -1;
                for (int g = 0; g < n_group; ++g)
                    if (!gtaken[g] && (best < 0 || gs[g] > gs[best])) best = g;
                gtaken[best] = 1;
            }
            for (int e = 0; e < E; ++e) allowed[e] = gtaken[e / gsize];
        }
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (allowed[e] && (best < 0 || c[e] > c[best])) best = e;
            allowed[best] = 0;
            topk_idx[(size_t)t * K + k] = best;
        }
        float sum = 0.0f;
        for (int k = 0; k < K; ++k) sum += s[topk_idx[(size_t)t * K + k]];
        for (int k = 0; k < K; ++k) {
            float v = s[topk_idx[(size_t)t * K + k]];
            if (normalize) v = v / sum;
            topk_w[(size_t)t * K + k] = v * scale;
        }
    }
    free(s); free(c); free(allowed); free(gs); free(gtaken);
    return ORACLE_OK;
}
