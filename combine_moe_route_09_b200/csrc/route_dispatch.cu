// Router top-K gating, the dispatch layout and the dispatch in ONE cooperative
// launch, for batches whose share per SM fits in shared memory.
//
// "Efficient and portable mixture-of-experts communication": Introduction
// (top-K experts per token, weights from the router's distribution), Portable
// Kernels (experts in blocks of E/R, a fixed region per (rank, expert)) and
// Dispatch (tokens of one expert contiguous, with their block scaling factors;
// the source of each row kept for the combine).  "MoonEP developer guide",
// core API example: tokens_per_expert, cu_seqlens, token_padding.
//
// The three steps give exactly the results of moe_route_topk,
// moe_dispatch_layout and moe_dispatch (the same per-row router, the same
// stable counting sort, the same FP8 arithmetic); what changes is when the
// bytes move.  The token rows x do not depend on the routing, so they are read
// (and quantised) while the router runs, and kept in shared memory until their
// slots are known; the rows then leave as TMA bulk stores.  One CTA per SM,
// all co-resident (cooperative launch); CTA b owns the contiguous tokens
// [S*b/G, S*(b+1)/G).  The host takes this kernel only for small shares
// (FP8: at most RD_FP8_MAX_TOKENS tokens per CTA), where the exchange and the
// quantiser cost less than the separate kernels' launches and round trips.
//
// Warp roles:
//   producer (warp 0)    waits until the routing warps hold their first logits,
//                        then bulk-loads each token's x row into the resident
//                        region (at most `inflight` rows in flight)
//   all 16 other warps   route the CTA's tokens (one warp per token); the
//                        experts and weights go to shared memory
//   quantisers (1..8)    FP8 only, in groups of P warps per token: turn token
//                        j's raw row into its resident slot j (codes, then the
//                        block scales); with at most 2 tokens per CTA they
//                        start once the routers have published the CTA's counts
//   routers (9..16)      rank the CTA's (token, k) pairs by expert, publish
//                        the CTA's histogram row and arrival mark, wait for
//                        every CTA's mark, compute the offsets and slots,
//                        write the layout and gating outputs, then issue the K
//                        bulk stores of each resident token once it is final
//
// The resident region has Qs slots of qrow bytes (FP8: codes + scales of one
// token).  A raw row needs rho slots (bf16 input: 2, fp32: 4).  Raw rows are
// placed in waves so that no raw row is overwritten before it is read and no
// finished slot is overwritten at all: wave w starts at token a_w and places
// raw row j at slot a_w + rho (j - a_w), as many rows as fit below Qs; slot j
// is written only once token j's raw row is in registers, and every raw row j
// lies at slots >= j.  With Qs = M + rho - 1 every token of a CTA with M
// tokens finds a window.  Before a raw row is loaded into a window, the last
// token whose raw row covered that window must be done (its mbarrier); before
// a quantiser group writes slot j, the token whose raw row last covered slot
// j must be done too (the groups run tokens out of order).
//
// Every wait is bounded (mbarriers and the arrival-mark poll); a timeout sets
// MOE_STATUS_TIMEOUT and every role leaves its loop; loads in flight are
// waited for (bounded) before the CTA exits.
#include "common.cuh"
#include "fp8_core.cuh"
#include "kernels.cuh"
#include "layout_core.cuh"
#include "route_core.cuh"
#include "tma.cuh"

namespace moe {

constexpr int RD_QUANT_WARPS = 8;
constexpr int RD_ROUTER_WARPS = 8;
constexpr int RD_WARPS = 1 + RD_QUANT_WARPS + RD_ROUTER_WARPS;
constexpr int RD_THREADS = RD_WARPS * 32;
constexpr int RD_QT = RD_QUANT_WARPS * 32;   // quantiser threads
constexpr int RD_RT = RD_ROUTER_WARPS * 32;  // router threads
constexpr int RD_MAX_ITERS = 8;              // FP8: one warp takes a row in <= 8 x 64 units (H <= 8192)
constexpr int RD_MAX_E = 512;
// FP8 rows are quantised inside the fused kernel only up to this many tokens per
// CTA.  The bit-exact quantiser costs about 1.2k cycles per 1024 channels and
// warp; with more tokens per SM that work is better hidden behind the many
// stores of the separate dispatch kernel (measured on the 4096 x 7168 prefill:
// one fused kernel took 117 us where route + layout + dispatch take 75 us).
constexpr int RD_FP8_MAX_TOKENS = 4;
constexpr int RD_BAR_R = 2;                  // named barrier of the routers (id 1 is not used)
constexpr int RD_BAR_ROUTED = 3;             // quantisers arrive, routers wait: routing complete
constexpr int RD_BAR_GROUP0 = 4;             // 4 .. 11: quantiser groups
constexpr int RD_BAR_PUBLISHED = 12;         // routers arrive once the CTA's counts are out, quantisers wait
constexpr long long RD_INFLIGHT_BYTES = 64 * 1024;  // token-row bytes a CTA keeps in flight

struct RdArgs {
    const float *logits;
    const uint8_t *x;
    int32_t *topk_idx;
    float *topk_w;
    int32_t *counts, *offsets, *rank_offsets, *slot_of, *row_src;
    uint8_t *xd;
    float *xs;
    LayoutHeader *hdr;
    unsigned *arrived;  // [G] epoch of the call once the CTA's histogram row is published
    uint16_t *hist;     // [G][Ep] per-CTA expert counts
    int32_t *status;
    int64_t cap;
    int S, H, E, K, R, P;
    int esz;         // input element bytes (2 or 4)
    int quant;       // 1: FP8 e4m3 with 128-channel scales; 0: copy
    int scale_bulk;  // FP8: the scale row is whole 16-byte units at 16-byte aligned addresses
    int Ep;          // E rounded up to a multiple of 8 (hist row stride: 16-byte rows of uint16)
    int inflight;    // raw rows a CTA keeps in flight at most
    int qgroup;      // quantiser warps per token (1, 2, 4 or 8)
    int qdelay;      // FP8: the quantisers start once the routers have published the CTA's counts
    int M;           // tokens per CTA at most
    int qrow;        // bytes of one resident slot (multiple of 16)
    int rho;         // slots covered by one raw row
    int Qs;          // slots in the resident region
    // dynamic shared memory offsets in bytes (the region starts at 0)
    int off_full, off_done, off_occ, off_pos, off_pe, off_pw, off_prk, off_sl, off_whist, off_tot, off_below, off_cnt,
        off_off, off_flag;
};

__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

template <int NPER>
__global__ void __launch_bounds__(RD_THREADS, 1) route_dispatch_kernel(const RdArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *const full = reinterpret_cast<uint64_t *>(smem + a.off_full);  // [M] raw row j landed
    uint64_t *const done = reinterpret_cast<uint64_t *>(smem + a.off_done);  // [M] resident slot j final
    uint64_t *const lg_in = reinterpret_cast<uint64_t *>(smem + a.off_flag + 8);  // routers hold their logits
    int *const occ = reinterpret_cast<int *>(smem + a.off_occ);              // [Qs] last raw row on the slot
    int *const pos = reinterpret_cast<int *>(smem + a.off_pos);              // [M] slot of raw row j
    int *const pe = reinterpret_cast<int *>(smem + a.off_pe);                // [M*K] expert of pair p
    int *const prk = reinterpret_cast<int *>(smem + a.off_prk);              // [M*K] rank of p in the CTA
    float *const pw = reinterpret_cast<float *>(smem + a.off_pw);            // [M*K] gating weight of pair p
    int *const sl = reinterpret_cast<int *>(smem + a.off_sl);                // [M*K] dispatched row of p
    uint16_t *const whist = reinterpret_cast<uint16_t *>(smem + a.off_whist);  // [RD_ROUTER_WARPS][E+2]
    int *const s_tot = reinterpret_cast<int *>(smem + a.off_tot);            // [E] pairs of e in all CTAs
    int *const s_below = reinterpret_cast<int *>(smem + a.off_below);        // [E] ... in the CTAs below
    int *const s_cnt = reinterpret_cast<int *>(smem + a.off_cnt);            // [E] ... in this CTA
    int *const s_off = reinterpret_cast<int *>(smem + a.off_off);            // [E+1] padded offsets
    volatile int *const s_abort = reinterpret_cast<volatile int *>(smem + a.off_flag);
    __shared__ unsigned s_epoch;
    __shared__ int s_wsum[RD_ROUTER_WARPS];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x, G = gridDim.x;
    const int t0 = (int)((long long)a.S * b / G), t1 = (int)((long long)a.S * (b + 1) / G);
    const int n = t1 - t0;
    const int K = a.K, E = a.E, WS = E + 2;
    const int row_bytes = a.H * a.esz;
    const uint32_t region = smem_addr(smem);
    const uint32_t full0 = smem_addr(full), done0 = smem_addr(done);

    if (tid == 0) {
        for (int j = 0; j < n; ++j) {
            mbar_init(full0 + 8u * j, 1);
            mbar_init(done0 + 8u * j, a.qgroup);
        }
        mbar_init(smem_addr(lg_in), RD_QUANT_WARPS + RD_ROUTER_WARPS);
        fence_mbar_init();
        *s_abort = 0;
    }
    for (int i = tid; i < a.Qs; i += RD_THREADS) occ[i] = -1;
    for (int i = tid; i < RD_ROUTER_WARPS * WS; i += RD_THREADS) whist[i] = 0;
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------- producer -------------------------------
        if (lane == 0) {
            int issued = 0;
            int aw = 0, wend = 0;  // the current wave: tokens [aw, wend)
            // The router's logits go first: its loads would otherwise queue behind
            // the token rows, and every later step of the layout waits for it.
            if (!mbar_wait(smem_addr(lg_in), 0, a.status)) *s_abort = 1;
            for (int j = 0; j < n; ++j) {
                if (*s_abort) break;
                // at most `inflight` rows in flight: deep enough to stream, shallow
                // enough that the layout's own round trips do not wait behind them
                if (j >= a.inflight && !mbar_wait(full0 + 8u * (j - a.inflight), 0, a.status)) {
                    *s_abort = 1;
                    break;
                }
                int p = j;
                if (a.quant) {
                    if (j == wend) {
                        aw = j;
                        wend = min(n, j + (a.Qs - j) / a.rho);
                    }
                    p = aw + a.rho * (j - aw);
                    int m = -1;
                    for (int q = p; q < p + a.rho; ++q) m = max(m, occ[q]);
                    if (m >= 0 && !mbar_wait(done0 + 8u * m, 0, a.status)) {
                        *s_abort = 1;
                        break;
                    }
                    for (int q = p; q < p + a.rho; ++q) occ[q] = j;
                }
                pos[j] = p;
                const uint32_t bar = full0 + 8u * j;
                mbar_arrive_expect_tx(bar, (uint32_t)row_bytes);
                bulk_g2s(region + (uint32_t)p * (uint32_t)a.qrow, a.x + (size_t)(t0 + j) * row_bytes,
                         (uint32_t)row_bytes, bar);
                ++issued;
            }
            // never leave a copy in flight when the CTA exits
            for (int j = 0; j < issued; ++j) mbar_wait(full0 + 8u * j, 0, a.status);
        }
        return;
    }

    // --------------- routing: all 16 compute warps, tokens cw, cw + 16, ... ---------------
    // The logits of each warp's first PF tokens are loaded before any token row
    // (the producer waits for lg_in); the experts and weights go to shared
    // memory (pe, pw) and reach global memory after the exchange below.
    {
        const int cw = warp - 1;
        constexpr int CW = RD_QUANT_WARPS + RD_ROUTER_WARPS;
        // this call's arrival mark: the generation (final once the previous
        // kernel on the stream is complete) plus one; loaded now, used later
        const bool first_router = tid == 32 * (1 + RD_QUANT_WARPS);
        const unsigned gen = first_router ? *(volatile unsigned *)&a.hdr->gen : 0u;
        constexpr int PF = NPER <= 8 ? 2 : 1;
        uint32_t key[PF][NPER];
        uint32_t dep = 0;
#pragma unroll
        for (int q = 0; q < PF; ++q) {
            const int i = cw + q * CW;
            if (i < n) {
                load_route_keys<NPER>(a.logits + (size_t)(t0 + i) * E, E, lane, key[q]);
#pragma unroll
                for (int j = 0; j < NPER; ++j) dep |= key[q][j];
            }
        }
        asm volatile("" ::"r"(dep));  // the loads have landed before the arrival below
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(lg_in));
        auto finish = [&](int i, uint32_t(&kk)[NPER]) {
            int e;
            float w;
            topk_softmax<NPER>(kk, K, lane, e, w);
            if (lane < K) {
                pe[i * K + lane] = e;
                pw[i * K + lane] = w;
            }
        };
#pragma unroll
        for (int q = 0; q < PF; ++q) {
            const int i = cw + q * CW;
            if (i < n) finish(i, key[q]);
        }
        for (int i = cw + PF * CW; i < n; i += CW) {
            uint32_t kk[NPER];
            load_route_keys<NPER>(a.logits + (size_t)(t0 + i) * E, E, lane, kk);
            finish(i, kk);
        }
        if (first_router) s_epoch = gen + 1u;
    }

    if (warp <= RD_QUANT_WARPS) {
        named_bar_arrive(RD_BAR_ROUTED, RD_QT + RD_RT);  // this warp's routing is in pe / pw
        // ------------------------------- quantisers -------------------------------
        // The 8 quantiser warps form groups of P (P = 1 when a CTA has 8 or more
        // tokens, up to 8 for a single token); group g turns tokens g, g + 8/P,
        // ... into their resident slots.  An iteration takes 64 P consecutive
        // 16-channel units (two per lane, independent chains), all of them read
        // before any of its codes is written; the codes of an iteration cover raw
        // bytes of units already read (the raw row may start at the token's own
        // slot), and the block scales, which lie past the codes, go in after the
        // last iteration.  Before writing slot j the group waits for the token
        // whose raw row last covered that slot.
        if (!a.quant) return;
        // With few tokens per CTA the quantisers are off the critical path, which
        // runs through the routers' ranking and the exchange: keeping the SM's
        // issue slots for the routers until their counts are published shortens it.
        if (a.qdelay) named_bar(RD_BAR_PUBLISHED, RD_QT + RD_RT);
        const int qw = warp - 1;
        const int P = a.qgroup, NG = RD_QUANT_WARPS / P;
        const int g = qw / P, gm = qw - g * P;
        const int gbar = RD_BAR_GROUP0 + g;
        auto gsync = [&]() {
            if (P > 1) named_bar(gbar, 32 * P);
            else __syncwarp();
        };
        auto gall = [&](bool v) { return P > 1 ? named_bar_and(gbar, 32 * P, v) : (bool)__all_sync(FULL, v); };
        const int units = a.H >> 4;  // a multiple of 8 (H % 128 == 0)
        const int span = 64 * P;
        const int iters = (units + span - 1) / span;
        const bool lead = (lane & 7) == 0;
        for (int j = g; j < n; j += NG) {
            bool ok = !*s_abort && mbar_wait(full0 + 8u * j, 0, a.status);
            const int m = occ[j];
            if (ok && m >= 0 && m != j) ok = mbar_wait(done0 + 8u * m, 0, a.status);
            if (!gall(ok)) {
                *s_abort = 1;
                break;
            }
            const uint32_t raw = region + (uint32_t)pos[j] * (uint32_t)a.qrow;
            const uint32_t dst = region + (uint32_t)j * (uint32_t)a.qrow;
            float sc[RD_MAX_ITERS][2];
#pragma unroll
            for (int it = 0; it < RD_MAX_ITERS; ++it) {
                if (it >= iters) break;
                const int u0 = it * span + gm * 64 + lane;
                float f[2][16];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int u = u0 + 32 * h;
                    if (u < units) {
                        if (a.esz == 4) {
                            const uint32_t src = raw + (uint32_t)u * 64u;
#pragma unroll
                            for (int l = 0; l < 4; ++l) {
                                const U4 v = lds128(src + 16u * l);
                                f[h][4 * l + 0] = __uint_as_float(v.x);
                                f[h][4 * l + 1] = __uint_as_float(v.y);
                                f[h][4 * l + 2] = __uint_as_float(v.z);
                                f[h][4 * l + 3] = __uint_as_float(v.w);
                            }
                        } else {
                            // lanes 32 bytes apart: lanes 4-7 (mod 8) read their upper half
                            // first, so each phase's eight 16-byte reads hit distinct banks
                            const uint32_t src = raw + (uint32_t)u * 32u;
                            const uint32_t sw = (uint32_t)(lane >> 2) & 1u;
                            const U4 a0 = lds128(src + 16u * sw), a1 = lds128(src + 16u * (sw ^ 1u));
                            const U4 v2[2] = {sw ? a1 : a0, sw ? a0 : a1};
#pragma unroll
                            for (int l = 0; l < 2; ++l) {
                                const U4 &v = v2[l];
                                f[h][8 * l + 0] = bf16lo(v.x); f[h][8 * l + 1] = bf16hi(v.x);
                                f[h][8 * l + 2] = bf16lo(v.y); f[h][8 * l + 3] = bf16hi(v.y);
                                f[h][8 * l + 4] = bf16lo(v.z); f[h][8 * l + 5] = bf16hi(v.z);
                                f[h][8 * l + 6] = bf16lo(v.w); f[h][8 * l + 7] = bf16hi(v.w);
                            }
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) f[h][e] = 0.f;
                    }
                }
                gsync();  // every raw read of this iteration, in the whole group, precedes its writes
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float m8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) m8[e] = fmaxf(fabsf(f[h][2 * e]), fabsf(f[h][2 * e + 1]));
#pragma unroll
                    for (int e = 0; e < 4; ++e) m8[e] = fmaxf(m8[e], m8[e + 4]);
                    float amax = fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3]));
                    amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
                    amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
                    amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 4));
                    sc[it][h] = scale_of(amax);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int u = u0 + 32 * h;
                    if (u < units) sts128(dst + (uint32_t)u * 16u, quant16(f[h], sc[it][h]));
                }
            }
            gsync();  // every raw read of the token precedes the scale writes
#pragma unroll
            for (int it = 0; it < RD_MAX_ITERS; ++it) {
                if (it >= iters) break;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int u = it * span + gm * 64 + lane + 32 * h;
                    if (u < units && lead) sts_f32(dst + (uint32_t)a.H + (uint32_t)(u >> 3) * 4u, sc[it][h]);
                }
            }
            fence_proxy_async_smem();  // the bulk stores (async proxy) read these bytes
            __syncwarp();
            if (lane == 0) mbar_arrive(done0 + 8u * j);
        }
        return;
    }

    // --------------------------------- routers ---------------------------------
    named_bar(RD_BAR_ROUTED, RD_QT + RD_RT);  // every compute warp's routing is in pe / pw
    const int rt = tid - 32 * (1 + RD_QUANT_WARPS), wr = rt >> 5;

    // ---- rank the CTA's pairs by expert, in ascending pair order ----
    const int np = n * K;
    const int nchunk = (np + 31) >> 5;
    const int cpw = (nchunk + RD_ROUTER_WARPS - 1) / RD_ROUTER_WARPS;
    const int c0 = wr * cpw, c1 = min(nchunk, c0 + cpw);
    const int nbits = expert_bits(E);
    const unsigned lt = lanemask_lt();
    for (int c = c0; c < c1; ++c) {
        const int p = c * 32 + lane;
        const int e = p < np ? pe[p] : -1;
        const unsigned peers = expert_peers(e, nbits);
        const int before = e >= 0 ? (int)whist[wr * WS + e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) whist[wr * WS + e] = (uint16_t)(before + __popc(peers));
        __syncwarp();
        if (p < np) prk[p] = before + __popc(peers & lt);
    }
    named_bar(RD_BAR_R, RD_RT);
    // per expert: exclusive prefix over the router warps, and the CTA's count
    for (int e = rt; e < E; e += RD_RT) {
        int run = 0;
#pragma unroll
        for (int ww = 0; ww < RD_ROUTER_WARPS; ++ww) {
            const int c = whist[ww * WS + e];
            whist[ww * WS + e] = (uint16_t)run;
            run += c;
        }
        s_cnt[e] = run;
        s_tot[e] = 0;
        s_below[e] = 0;
    }
    named_bar(RD_BAR_R, RD_RT);
    for (int e = rt; e < a.Ep; e += RD_RT) a.hist[(size_t)b * a.Ep + e] = (uint16_t)(e < E ? s_cnt[e] : 0);
    for (int c = c0; c < c1; ++c) {
        const int p = c * 32 + lane;
        if (p < np) prk[p] += whist[wr * WS + pe[p]];
    }
    // ---- one exchange: publish the histogram row, mark arrival, wait for every CTA ----
    __threadfence();
    named_bar(RD_BAR_R, RD_RT);
    const unsigned epoch = s_epoch;
    if (rt == 0) *(volatile unsigned *)&a.arrived[b] = epoch;
    if (a.quant && a.qdelay) named_bar_arrive(RD_BAR_PUBLISHED, RD_QT + RD_RT);  // the quantisers may start
    bool layout_ok = true;
    {
        const unsigned long long t_start = globaltimer();
        for (;;) {
            bool mine = true;
            for (int i = rt; i < G; i += RD_RT) mine &= *(volatile const unsigned *)&a.arrived[i] == epoch;
            // both decisions are taken by all router threads together (barrier reductions)
            if (named_bar_and(RD_BAR_R, RD_RT, mine)) break;
            if (!named_bar_and(RD_BAR_R, RD_RT, globaltimer() - t_start <= MOE_WAIT_NS)) {
                if (rt == 0) set_status(a.status, MOE_STATUS_TIMEOUT);
                layout_ok = false;
                break;
            }
            __nanosleep(32);
        }
    }
    __threadfence();
    if (!layout_ok) *s_abort = 1;
    // every CTA has read the generation before it marked its arrival: the next call's mark
    if (layout_ok && b == 0 && rt == 0) *(volatile unsigned *)&a.hdr->gen = epoch;

    if (layout_ok) {
        // ---- per expert: pairs in the CTAs below this one and in all CTAs ----
        // rows are read 16 bytes (8 experts) at a time, all loads of a batch in
        // flight together; thread = (column group, first row), rows step by rstep
        const int cgN = a.Ep >> 3;
        const int rstep = RD_RT / cgN;  // >= 4 for E <= 512
        const int cg = rt % cgN, r0 = rt / cgN;
        int bl[8] = {0, 0, 0, 0, 0, 0, 0, 0}, to[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (r0 < rstep) {
            const int4 *col = reinterpret_cast<const int4 *>(a.hist) + cg;
            constexpr int BATCH = 16;
            for (int rb = r0; rb < G; rb += BATCH * rstep) {
                int4 v[BATCH];
#pragma unroll
                for (int q = 0; q < BATCH; ++q) {
                    const int r = rb + q * rstep;
                    v[q] = r < G ? __ldcg(col + (size_t)r * cgN) : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int q = 0; q < BATCH; ++q) {
                    const int r = rb + q * rstep;
                    const uint32_t u[4] = {(uint32_t)v[q].x, (uint32_t)v[q].y, (uint32_t)v[q].z, (uint32_t)v[q].w};
                    const bool below = r < b;
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int lo = (int)(u[h] & 0xffffu), hi = (int)(u[h] >> 16);
                        to[2 * h] += lo;
                        to[2 * h + 1] += hi;
                        if (below) {
                            bl[2 * h] += lo;
                            bl[2 * h + 1] += hi;
                        }
                    }
                }
            }
            const int e0 = cg * 8;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (e0 + q < E) {
                    atomicAdd(&s_below[e0 + q], bl[q]);
                    atomicAdd(&s_tot[e0 + q], to[q]);
                }
            }
        }
        named_bar(RD_BAR_R, RD_RT);
        // ---- exclusive scan of the padded counts over experts (4 per thread) ----
        int pc[4], sum = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = 4 * rt + q;
            pc[q] = e < E ? pad_count(s_tot[e], a.P) : 0;
            sum += pc[q];
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += o;
        }
        if (lane == 31) s_wsum[wr] = incl;
        named_bar(RD_BAR_R, RD_RT);
        if (wr == 0) {
            int v = lane < RD_ROUTER_WARPS ? s_wsum[lane] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(FULL, v, off);
                if (lane >= off) v += o;
            }
            if (lane < RD_ROUTER_WARPS) s_wsum[lane] = v;  // inclusive over warps
        }
        named_bar(RD_BAR_R, RD_RT);
        int base = incl - sum + (wr > 0 ? s_wsum[wr - 1] : 0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = 4 * rt + q;
            if (e < E) s_off[e] = base;
            base += pc[q];
        }
        if (rt == 0) s_off[E] = s_wsum[RD_ROUTER_WARPS - 1];
        named_bar(RD_BAR_R, RD_RT);
        if (b == 0) {
            for (int e = rt; e <= E; e += RD_RT) a.offsets[e] = s_off[e];
            for (int e = rt; e < E; e += RD_RT) a.counts[e] = s_tot[e];
            const int Eloc = E / a.R;
            for (int r = rt; r <= a.R; r += RD_RT) a.rank_offsets[r] = s_off[r * Eloc];
            if (rt == 0 && (int64_t)s_off[E] > a.cap) set_status(a.status, MOE_STATUS_OVERFLOW);
        }
        // ---- slots: offset of the expert + pairs of it in lower CTAs + rank in this CTA ----
        bool over = false;
        const int pbase = t0 * K;
        for (int p = rt; p < np; p += RD_RT) {
            const int e = pe[p];
            int s = s_off[e] + s_below[e] + prk[p];
            if ((int64_t)s >= a.cap) {
                s = -1;
                over = true;
            }
            sl[p] = s;
            a.slot_of[(size_t)pbase + p] = s;
            if (s >= 0) a.row_src[s] = pbase + p;
        }
        if (over) set_status(a.status, MOE_STATUS_OVERFLOW);
        // ---- the gating outputs of this CTA's tokens ----
        for (int p = rt; p < np; p += RD_RT) {
            a.topk_idx[(size_t)pbase + p] = pe[p];
            a.topk_w[(size_t)pbase + p] = pw[p];
        }
        // ---- padding rows (a warp per expert, spread over the CTAs) and rows past the layout ----
        for (int e = b * RD_ROUTER_WARPS + wr; e < E; e += G * RD_ROUTER_WARPS) {
            const int64_t lo = (int64_t)s_off[e] + s_tot[e];
            int64_t hi = s_off[e + 1];
            if (hi > a.cap) hi = a.cap;
            for (int64_t r = lo + lane; r < hi; r += 32) a.row_src[r] = -1;
        }
        for (int64_t r = (int64_t)s_off[E] + (int64_t)b * RD_RT + rt; r < a.cap; r += (int64_t)G * RD_RT)
            a.row_src[r] = -1;
        named_bar(RD_BAR_R, RD_RT);

        // ---- scatter: each token's K copies leave as bulk stores once it is resident ----
        const int nb = a.H >> 7;
        for (int i = wr; i < n; i += RD_ROUTER_WARPS) {
            const uint32_t ready = (a.quant ? done0 : full0) + 8u * i;
            if (!__all_sync(FULL, mbar_wait(ready, 0, a.status))) {
                *s_abort = 1;
                break;
            }
            if (lane < K) {
                const int s = sl[i * K + lane];
                if (s >= 0) {
                    const uint32_t src = region + (uint32_t)i * (uint32_t)a.qrow;
                    if (a.quant) {
                        bulk_s2g(a.xd + (size_t)s * a.H, src, (uint32_t)a.H);
                        if (a.scale_bulk) {
                            bulk_s2g(a.xs + (size_t)s * nb, src + (uint32_t)a.H, (uint32_t)nb * 4u);
                        } else {
                            for (int q = 0; q < nb; ++q)
                                a.xs[(size_t)s * nb + q] = lds_f32(src + (uint32_t)a.H + 4u * q);
                        }
                    } else {
                        bulk_s2g(a.xd + (size_t)s * row_bytes, src, (uint32_t)row_bytes);
                    }
                }
            }
        }
    }
    bulk_commit();
    bulk_wait_all();  // the stores have read the region before the CTA exits
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------

// Workspace of the fused kernel: the layout's own workspace first (so the two
// calls can share one buffer without touching each other's state), then the
// arrival marks [RD_MAX_CTAS] and the histogram rows [RD_MAX_CTAS][Ep] uint16.
static size_t rd_marks_offset(int S, int E, int K) { return (layout_workspace_bytes(S, E, K) + 255) / 256 * 256; }
static int rd_row(int E) { return (E + 7) / 8 * 8; }

size_t route_dispatch_workspace_bytes(int S, int E, int K) {
    return rd_marks_offset(S, E, K) + 4 * (size_t)RD_MAX_CTAS + 2 * (size_t)RD_MAX_CTAS * rd_row(E);
}

// Plans the fused launch for these sizes on the current device: false if it
// does not apply (then the caller runs the three separate kernels).
static cudaError_t rd_plan(int S, int H, int E, int K, int R, int P, int dtype, int quant, RdArgs *a, size_t *smem,
                           int *grid, bool *ok) {
    *ok = false;
    if (S < 1 || E > RD_MAX_E || K > E || H < 1) return cudaSuccess;
    const int esz = dtype == MOE_DTYPE_F32 ? 4 : 2;
    if (quant && (H % 128 != 0 || H > RD_MAX_ITERS * 64 * 16)) return cudaSuccess;
    const long long row_bytes = (long long)H * esz;
    if (row_bytes >= (1 << 20)) return cudaSuccess;  // one mbarrier transaction per row
    int dev = 0, sms = 0, max_optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    // one CTA per SM; FP8 batches smaller than two tokens per SM use half as many
    // CTAs (two tokens each): the exchange costs less with fewer CTAs, and the
    // quantiser groups still split each token (measured on a 128-token decode
    // batch: 10.4 us with 64 CTAs against 11.4 us with 128)
    int G = quant ? (S + 1) / 2 : S;
    if (G > sms) G = sms;
    if (G > RD_MAX_CTAS) G = RD_MAX_CTAS;
    if (G < 1) return cudaSuccess;
    const int M = (S + G - 1) / G;
    if (quant && M > RD_FP8_MAX_TOKENS) return cudaSuccess;
    const int qrow = quant ? (H + (H / 128) * 4 + 15) / 16 * 16 : (int)row_bytes;
    const int rho = quant ? (int)((row_bytes + qrow - 1) / qrow) : 1;
    const int Qs = quant ? M + rho - 1 : M;
    auto al = [](size_t v, size_t q) { return (v + q - 1) / q * q; };
    size_t off = (size_t)Qs * qrow;
    a->off_full = (int)(off = al(off, 16));
    off += 8 * (size_t)M;
    a->off_done = (int)off;
    off += 8 * (size_t)M;
    a->off_occ = (int)off;
    off += 4 * (size_t)Qs;
    a->off_pos = (int)off;
    off += 4 * (size_t)M;
    a->off_pe = (int)off;
    off += 4 * (size_t)M * K;
    a->off_pw = (int)off;
    off += 4 * (size_t)M * K;
    a->off_prk = (int)off;
    off += 4 * (size_t)M * K;
    a->off_sl = (int)off;
    off += 4 * (size_t)M * K;
    a->off_whist = (int)off;
    off += al(2 * (size_t)RD_ROUTER_WARPS * (E + 2), 4);
    a->off_tot = (int)off;
    off += 4 * (size_t)E;
    a->off_below = (int)off;
    off += 4 * (size_t)E;
    a->off_cnt = (int)off;
    off += 4 * (size_t)E;
    a->off_off = (int)off;
    off += 4 * (size_t)(E + 1);
    a->off_flag = (int)(off = al(off, 16));
    off += 16;
    // the kernel's static shared memory (the warp sums, 128 bytes) comes on top
    if (off + 256 > (size_t)max_optin) return cudaSuccess;
    a->S = S;
    a->H = H;
    a->E = E;
    a->K = K;
    a->R = R;
    a->P = P;
    a->esz = esz;
    a->quant = quant ? 1 : 0;
    a->Ep = rd_row(E);
    a->qgroup = M >= 8 ? 1 : (M >= 4 ? 2 : (M >= 2 ? 4 : 8));
    a->qdelay = quant && M <= 2 ? 1 : 0;
    a->inflight = (int)(RD_INFLIGHT_BYTES / row_bytes > 1 ? RD_INFLIGHT_BYTES / row_bytes : 1);
    a->M = M;
    a->qrow = qrow;
    a->rho = rho;
    a->Qs = Qs;
    *smem = off;
    *grid = G;
    *ok = true;
    return cudaSuccess;
}

template <int NPER>
static cudaError_t rd_launch(const RdArgs &a, size_t smem, int grid, cudaStream_t st, bool *launched, bool dry) {
    *launched = false;
    static KernelSlots<decltype(&route_dispatch_kernel<NPER>)> slots;
    int sms = 0, per_sm = 0;
    cudaError_t e = slots.prepare(&route_dispatch_kernel<NPER>, RD_THREADS, smem, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    if ((long long)sms * per_sm < grid) return cudaSuccess;  // not co-resident: separate kernels
    static PerDeviceFlag coop_ok, pdl_ok;
    if (!coop_ok.on()) return cudaSuccess;
    if (dry) {
        *launched = true;
        return cudaSuccess;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(RD_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_ok.on() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, route_dispatch_kernel<NPER>, a);
    if (e != cudaSuccess && cfg.numAttrs == 2) {
        (void)cudaGetLastError();  // the pair was refused: cooperative only on this device from now on
        pdl_ok.disable();
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, route_dispatch_kernel<NPER>, a);
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();  // no cooperative launch on this device: separate kernels from now on
        coop_ok.disable();
        return cudaSuccess;
    }
    *launched = true;
    return cudaSuccess;
}

static cudaError_t rd_try(RdArgs &a, size_t smem, int grid, cudaStream_t st, bool *launched, bool dry) {
    const int nper = (a.E + 31) / 32;
    if (nper <= 1) return rd_launch<1>(a, smem, grid, st, launched, dry);
    if (nper <= 2) return rd_launch<2>(a, smem, grid, st, launched, dry);
    if (nper <= 4) return rd_launch<4>(a, smem, grid, st, launched, dry);
    if (nper <= 8) return rd_launch<8>(a, smem, grid, st, launched, dry);
    if (nper <= 12) return rd_launch<12>(a, smem, grid, st, launched, dry);
    return rd_launch<16>(a, smem, grid, st, launched, dry);
}

int route_dispatch_kernel_count(int S, int H, int E, int K, int dtype, int quant) {
    RdArgs a = {};
    size_t smem = 0;
    int grid = 0;
    bool ok = false;
    if (rd_plan(S, H, E, K, 1, 0, dtype, quant, &a, &smem, &grid, &ok) != cudaSuccess) return -1;
    if (ok) {
        bool one = false;
        if (rd_try(a, smem, grid, nullptr, &one, true) != cudaSuccess) return -1;
        if (one) return 1;
    }
    const int lk = layout_kernel_count(S, E, K);
    return lk < 0 ? -1 : 2 + lk;
}

cudaError_t launch_route_dispatch(const float *logits, const void *x, int dtype, int S, int H, int E, int K, int R,
                                  int P, int quant, int32_t *topk_idx, float *topk_w, int32_t *counts,
                                  int32_t *offsets, int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src,
                                  void *xd, float *xs, int64_t cap, void *workspace, int32_t *status,
                                  cudaStream_t st, int sms) {
    if (S == 0) {
        // no tokens: the layout alone (zero counts, row_src = -1 everywhere)
        return launch_layout(topk_idx, 0, E, K, R, P, counts, offsets, rank_offsets, slot_of, row_src, cap,
                             workspace, status, st);
    }
    RdArgs a = {};
    size_t smem = 0;
    int grid = 0;
    bool ok = false;
    cudaError_t e = rd_plan(S, H, E, K, R, P, dtype, quant, &a, &smem, &grid, &ok);
    if (e != cudaSuccess) return e;
    if (ok) {
        a.logits = logits;
        a.x = reinterpret_cast<const uint8_t *>(x);
        a.topk_idx = topk_idx;
        a.topk_w = topk_w;
        a.counts = counts;
        a.offsets = offsets;
        a.rank_offsets = rank_offsets;
        a.slot_of = slot_of;
        a.row_src = row_src;
        a.xd = reinterpret_cast<uint8_t *>(xd);
        a.xs = xs;
        a.hdr = reinterpret_cast<LayoutHeader *>(workspace);
        char *const marks = reinterpret_cast<char *>(workspace) + rd_marks_offset(S, E, K);
        a.arrived = reinterpret_cast<unsigned *>(marks);
        a.hist = reinterpret_cast<uint16_t *>(marks + 4 * RD_MAX_CTAS);
        a.status = status;
        a.cap = cap;
        a.scale_bulk = (quant && (H / 128) % 4 == 0 && (reinterpret_cast<uintptr_t>(xs) & 15) == 0) ? 1 : 0;
        bool launched = false;
        e = rd_try(a, smem, grid, st, &launched, false);
        if (e != cudaSuccess || launched) return e;
    }
    // the separate kernels: same results
    e = launch_route_topk(logits, S, E, K, topk_idx, topk_w, st, sms);
    if (e != cudaSuccess) return e;
    e = launch_layout(topk_idx, S, E, K, R, P, counts, offsets, rank_offsets, slot_of, row_src, cap, workspace,
                      status, st);
    if (e != cudaSuccess) return e;
    return launch_dispatch(x, dtype, S, H, K, slot_of, quant, xd, xs, cap, status, st);
}

}  // namespace moe
