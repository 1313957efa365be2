// Per-expert histogram and prefix scan into the padded, expert-contiguous layout.
//
// "MoonEP developer guide", core API example and tuning parameters:
// tokens_per_expert, cu_seqlens, groups padded to token_padding rows.
// "Efficient and portable mixture-of-experts communication", Portable Kernels
// (a fixed receive bound per (rank, local expert); experts in blocks of E/R)
// and Dispatch (tokens of one expert contiguous; the source of each row kept
// for the combine).
//
// Layouts whose tile histograms every CTA can scan (T * E <= 64 Ki entries) and
// whose tiles fit one co-resident grid run as ONE cooperative kernel
// (layout_fused, below): ranks in registers, one bounded grid barrier, each CTA
// scanning the tile histograms itself.  Larger layouts use two kernels, with no
// spin-waits and no global atomics except one arrival counter:
//
//  layout_hist   one CTA per tile of LT_TILE pairs.  Each warp ranks its 32
//                pairs by expert (peers sharing an expert are found with one ballot per id bit;
//                the lowest peer adds the group size to the warp's private
//                shared-memory histogram), so the tile histogram is built
//                without atomics.  The CTA writes it to hist[tile][E], then
//                takes a ticket; the CTA with the last ticket (all tiles are
//                written by then) turns hist into per-expert exclusive prefixes
//                over tiles, pads the totals and scans them over experts into
//                counts / offsets / rank_offsets, and resets the ticket.
//  layout_slots  one CTA per tile again: recomputes the same per-warp ranks,
//                converts the per-warp histograms to prefixes over warps, and
//                writes slot = offsets[e] + tile prefix + warp prefix + rank,
//                then row_src, and -1 into padding rows and rows past offsets[E].
//
// The slot of a pair is therefore offsets[e] plus the number of earlier pairs
// (ascending t*K + k) with the same expert: a stable counting sort.
#include "common.cuh"
#include "kernels.cuh"
#include "layout_core.cuh"
#include "tma.cuh"

namespace moe {


__global__ void __launch_bounds__(LT_THREADS)
    layout_hist_kernel(const int32_t *__restrict__ topk_idx, int npairs, int E, int R, int P,
                       int64_t cap, int32_t *hist, LayoutHeader *hdr, int32_t *__restrict__ counts,
                       int32_t *__restrict__ offsets, int32_t *__restrict__ rank_offsets,
                       int32_t *status) {
    extern __shared__ uint16_t whist[];  // [LT_WARPS][E]
    __shared__ int s_part[1024];
    __shared__ int s_tot[1024];
    __shared__ int s_off[1025];
    __shared__ int s_wsum[LT_WARPS];
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int tile = blockIdx.x, T = gridDim.x;
    for (int i = tid; i < LT_WARPS * E; i += LT_THREADS) whist[i] = 0;
    pdl_wait();
    pdl_trigger();
    __syncthreads();

    bool bad = false;
    int ev[LT_ITEMS];  // all loads first, so their latencies overlap
#pragma unroll
    for (int it = 0; it < LT_ITEMS; ++it) {
        const int p = tile * LT_TILE + (w * LT_ITEMS + it) * 32 + lane;
        ev[it] = p < npairs ? __ldg(topk_idx + p) : -1;
    }
#pragma unroll
    for (int it = 0; it < LT_ITEMS; ++it) {
        const int p = tile * LT_TILE + (w * LT_ITEMS + it) * 32 + lane;
        int e = ev[it];
        if (p < npairs && (e < 0 || e >= E)) {
            bad = true;
            e = -1;
        }
        const unsigned peers = expert_peers(e, expert_bits(E));
        if (e >= 0 && lane == __ffs(peers) - 1) whist[w * E + e] += (uint16_t)__popc(peers);
        __syncwarp();
    }
    if (bad) set_status(status, MOE_STATUS_BAD_INDEX);
    __syncthreads();
    for (int e = tid; e < E; e += LT_THREADS) {
        int c = 0;
#pragma unroll
        for (int ww = 0; ww < LT_WARPS; ++ww) c += whist[ww * E + e];
        hist[(size_t)tile * E + e] = c;
    }
    // Publish this tile's histogram, then take a ticket; the last ticket scans.
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&hdr->ticket, 1u) == (unsigned)(T - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // (A) per-expert sums over groups of tiles; G groups run side by side.
    int G = LT_THREADS / E;
    if (G < 1) G = 1;
    if (G > T) G = T;
    const int tpg = (T + G - 1) / G;
    for (int idx = tid; idx < G * E; idx += LT_THREADS) {
        const int g = idx / E, e = idx - g * E;
        const int t1 = min(T, (g + 1) * tpg);
        int c = 0;
        for (int t = g * tpg; t < t1; t += 8) {
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = t + j < t1 ? __ldcg(hist + (size_t)(t + j) * E + e) : 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) c += v[j];
        }
        s_part[idx] = c;
    }
    __syncthreads();
    // (B) exclusive prefix over groups; totals per expert.
    for (int e = tid; e < E; e += LT_THREADS) {
        int run = 0;
        for (int g = 0; g < G; ++g) {
            const int c = s_part[g * E + e];
            s_part[g * E + e] = run;
            run += c;
        }
        s_tot[e] = run;
        counts[e] = run;
    }
    __syncthreads();
    // (C) exclusive prefix over tiles, in place in hist.
    for (int idx = tid; idx < G * E; idx += LT_THREADS) {
        const int g = idx / E, e = idx - g * E;
        const int t1 = min(T, (g + 1) * tpg);
        int run = s_part[idx];
        for (int t = g * tpg; t < t1; ++t) {
            const int c = __ldcg(hist + (size_t)t * E + e);
            hist[(size_t)t * E + e] = run;
            run += c;
        }
    }
    // (D) exclusive scan of the padded counts over experts: two experts per thread.
    const int e0 = 2 * tid, e1 = 2 * tid + 1;
    const int p0 = e0 < E ? pad_count(s_tot[e0], P) : 0;
    const int p1 = e1 < E ? pad_count(s_tot[e1], P) : 0;
    int incl = p0 + p1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_wsum[w] = incl;
    __syncthreads();
    if (w == 0) {
        int v = lane < LT_WARPS ? s_wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(FULL, v, off);
            if (lane >= off) v += o;
        }
        if (lane < LT_WARPS) s_wsum[lane] = v;  // inclusive over warps
    }
    __syncthreads();
    const int base = incl - (p0 + p1) + (w > 0 ? s_wsum[w - 1] : 0);
    if (e0 < E) s_off[e0] = base;
    if (e1 < E) s_off[e1] = base + p0;
    if (tid == 0) s_off[E] = s_wsum[LT_WARPS - 1];
    __syncthreads();
    for (int e = tid; e <= E; e += LT_THREADS) offsets[e] = s_off[e];
    const int Eloc = E / R;
    for (int r = tid; r <= R; r += LT_THREADS) rank_offsets[r] = s_off[r * Eloc];
    if (tid == 0) {
        if ((int64_t)s_off[E] > cap) set_status(status, MOE_STATUS_OVERFLOW);
        hdr->ticket = 0u;  // every other CTA has taken its ticket already
    }
}

__global__ void __launch_bounds__(LT_THREADS)
    layout_slots_kernel(const int32_t *__restrict__ topk_idx, int npairs, int E,
                        const int32_t *__restrict__ hist, const int32_t *__restrict__ counts,
                        const int32_t *__restrict__ offsets, int64_t cap,
                        int32_t *__restrict__ slot_of, int32_t *__restrict__ row_src,
                        int32_t *status) {
    extern __shared__ uint16_t whist[];  // [LT_WARPS][E]
    __shared__ int s_base[1024];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int tile = blockIdx.x;
    for (int i = tid; i < LT_WARPS * E; i += LT_THREADS) whist[i] = 0;
    __syncthreads();

    // Before pdl_wait: this kernel follows layout_hist in the same call, and
    // layout_hist triggered only after its own wait, so topk_idx (written two
    // launches back or earlier) is complete; layout_hist only reads it.  The
    // rank computation below therefore overlaps layout_hist's scan.  Loads go
    // through L2 (ld.global.cg), never a stale L1 line.
    int my_e[LT_ITEMS], my_r[LT_ITEMS];
    const unsigned lt = lanemask_lt();
    int ev[LT_ITEMS];  // all loads first, so their latencies overlap
#pragma unroll
    for (int it = 0; it < LT_ITEMS; ++it) {
        const int p = tile * LT_TILE + (w * LT_ITEMS + it) * 32 + lane;
        ev[it] = p < npairs ? __ldcg(topk_idx + p) : -1;
    }
#pragma unroll
    for (int it = 0; it < LT_ITEMS; ++it) {
        int e = ev[it];
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = expert_peers(e, expert_bits(E));
        const int before = e >= 0 ? (int)whist[w * E + e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) whist[w * E + e] = (uint16_t)(before + __popc(peers));
        __syncwarp();
        my_e[it] = e;
        my_r[it] = before + __popc(peers & lt);
    }
    __syncthreads();
    for (int e = tid; e < E; e += LT_THREADS) {
        int run = 0;
#pragma unroll
        for (int ww = 0; ww < LT_WARPS; ++ww) {
            const int c = whist[ww * E + e];
            whist[ww * E + e] = (uint16_t)run;
            run += c;
        }
    }
    pdl_wait();  // offsets, counts and the tile prefixes come from layout_hist
    pdl_trigger();
    for (int e = tid; e < E; e += LT_THREADS)
        s_base[e] = __ldcg(offsets + e) + __ldcg(hist + (size_t)tile * E + e);
    __syncthreads();

    bool over = false;
#pragma unroll
    for (int it = 0; it < LT_ITEMS; ++it) {
        const int p = tile * LT_TILE + (w * LT_ITEMS + it) * 32 + lane;
        if (p >= npairs) continue;
        const int e = my_e[it];
        int s = -1;
        if (e >= 0) {
            s = s_base[e] + whist[w * E + e] + my_r[it];
            if ((int64_t)s >= cap) {
                s = -1;
                over = true;
            }
        }
        slot_of[p] = s;
        if (s >= 0) row_src[s] = p;
    }
    if (over) set_status(status, MOE_STATUS_OVERFLOW);

    // Padding rows of each expert, one warp per expert.
    const int gw = tile * LT_WARPS + w, nw = gridDim.x * LT_WARPS;
    for (int e = gw; e < E; e += nw) {
        const int64_t lo = (int64_t)__ldcg(offsets + e) + __ldcg(counts + e);
        int64_t hi = __ldcg(offsets + e + 1);
        if (hi > cap) hi = cap;
        for (int64_t r = lo + lane; r < hi; r += 32) row_src[r] = -1;
    }
    // Rows past the layout.
    const int64_t tail0 = __ldcg(offsets + E);
    for (int64_t r = tail0 + (int64_t)tile * LT_THREADS + tid; r < cap;
         r += (int64_t)gridDim.x * LT_THREADS)
        row_src[r] = -1;
}

// ------------------------------------------------------------------------------------------
// Fused single-launch layout (cooperative grid; used when every CTA can read
// all tile histograms cheaply): phase 1 ranks the pairs of this CTA's tiles
// and publishes the tile histograms; one grid barrier; phase 2 has every CTA
// scan the tile histograms itself (its tiles' prefixes, the totals, the padded
// offsets) and write its slots.  The barrier's wait is time-bounded.
// ------------------------------------------------------------------------------------------

constexpr int LF_MAX_HIST = 64 * 1024;  // T * E entries a CTA may scan in phase 2

// Grid-wide barrier of the whole CTA (see grid_arrive_wait).
__device__ bool grid_barrier(LayoutHeader *hdr, int32_t *status) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) s_ok = grid_arrive_wait(hdr, status) ? 1 : 0;
    __syncthreads();
    return s_ok != 0;
}

// Ranks the 32 * LT_ITEMS pairs of warp w in tile `tile` by expert: my_e = expert
// (-1: none or invalid), my_r = rank among the warp's earlier pairs of that expert;
// whist[w][e] accumulates the warp's counts (whist must be zeroed).
__device__ __forceinline__ bool rank_tile(const int32_t *topk_idx, int npairs, int E, int tile, int w, int lane,
                                          uint16_t *whist, int (&my_e)[LT_ITEMS], int (&my_r)[LT_ITEMS]) {
    bool bad = false;
    const unsigned lt = lanemask_lt();
    int ev[LT_ITEMS];  // all loads first, so their latencies overlap
#pragma unroll
    for (int it = 0; it < LT_ITEMS; ++it) {
        const int p = tile * LT_TILE + (w * LT_ITEMS + it) * 32 + lane;
        ev[it] = p < npairs ? __ldcg(topk_idx + p) : -1;
    }
#pragma unroll
    for (int it = 0; it < LT_ITEMS; ++it) {
        const int p = tile * LT_TILE + (w * LT_ITEMS + it) * 32 + lane;
        int e = ev[it];
        if (p < npairs && (e < 0 || e >= E)) {
            bad = true;
            e = -1;
        }
        const unsigned peers = expert_peers(e, expert_bits(E));
        const int before = e >= 0 ? (int)whist[w * E + e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) whist[w * E + e] = (uint16_t)(before + __popc(peers));
        __syncwarp();
        my_e[it] = e;
        my_r[it] = before + __popc(peers & lt);
    }
    return bad;
}

__global__ void __launch_bounds__(LT_THREADS)
    layout_fused_kernel(const int32_t *__restrict__ topk_idx, int npairs, int E, int R, int P, int64_t cap,
                        int T, int32_t *hist, LayoutHeader *hdr, int32_t *__restrict__ counts,
                        int32_t *__restrict__ offsets, int32_t *__restrict__ rank_offsets,
                        int32_t *__restrict__ slot_of, int32_t *__restrict__ row_src, int32_t *status) {
    extern __shared__ __align__(16) uint8_t lf_smem[];
    uint16_t *whist = reinterpret_cast<uint16_t *>(lf_smem);                     // [LT_WARPS][E]
    int *s_all = reinterpret_cast<int *>(lf_smem + ((LT_WARPS * E * 2 + 15) & ~15));  // [G][E]
    int *s_below = s_all + 1024;                                                  // [G][E]
    __shared__ int s_tot[1024];
    __shared__ int s_base[1024];
    __shared__ int s_off[1025];
    __shared__ int s_wsum[LT_WARPS];

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    // this CTA's tiles [t0, t1): a contiguous, balanced share of the T tiles
    const int t0 = (int)((long long)T * blockIdx.x / gridDim.x);
    const int t1 = (int)((long long)T * (blockIdx.x + 1) / gridDim.x);
    const bool single = t1 - t0 == 1;
    pdl_wait();
    pdl_trigger();

    // ---- phase 1: tile histograms ----
    int my_e[LT_ITEMS], my_r[LT_ITEMS];
    bool bad = false;
    for (int tile = t0; tile < t1; ++tile) {
        for (int i = tid; i < LT_WARPS * E; i += LT_THREADS) whist[i] = 0;
        __syncthreads();
        bad |= rank_tile(topk_idx, npairs, E, tile, w, lane, whist, my_e, my_r);
        __syncthreads();
        for (int e = tid; e < E; e += LT_THREADS) {
            int cnt = 0;
#pragma unroll
            for (int ww = 0; ww < LT_WARPS; ++ww) cnt += whist[ww * E + e];
            hist[(size_t)tile * E + e] = cnt;
        }
        if (!single) __syncthreads();  // whist is rebuilt for the next tile
    }
    if (bad) set_status(status, MOE_STATUS_BAD_INDEX);
    __threadfence();
    if (!grid_barrier(hdr, status)) return;

    // ---- phase 2a: per expert, the sum over tiles below t0 and over all tiles ----
    int G = LT_THREADS / E;
    if (G < 1) G = 1;
    if (G > T) G = T;
    const int tpg = (T + G - 1) / G;
    for (int idx = tid; idx < G * E; idx += LT_THREADS) {
        const int g = idx / E, e = idx - g * E;
        const int ta = g * tpg, tb = min(T, ta + tpg);
        int all = 0, below = 0;
        for (int tt = ta; tt < tb; tt += 8) {
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = tt + j < tb ? __ldcg(hist + (size_t)(tt + j) * E + e) : 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                all += v[j];
                below += tt + j < t0 ? v[j] : 0;
            }
        }
        s_all[idx] = all;
        s_below[idx] = below;
    }
    __syncthreads();
    for (int e = tid; e < E; e += LT_THREADS) {
        int all = 0, below = 0;
        for (int g = 0; g < G; ++g) {
            all += s_all[g * E + e];
            below += s_below[g * E + e];
        }
        s_tot[e] = all;
        s_base[e] = below;
    }
    __syncthreads();
    // ---- phase 2b: exclusive scan of the padded counts over experts, two per thread ----
    const int e0 = 2 * tid, e1 = 2 * tid + 1;
    const int p0 = e0 < E ? pad_count(s_tot[e0], P) : 0;
    const int p1 = e1 < E ? pad_count(s_tot[e1], P) : 0;
    int incl = p0 + p1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_wsum[w] = incl;
    __syncthreads();
    if (w == 0) {
        int v = lane < LT_WARPS ? s_wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(FULL, v, off);
            if (lane >= off) v += o;
        }
        if (lane < LT_WARPS) s_wsum[lane] = v;
    }
    __syncthreads();
    const int base = incl - (p0 + p1) + (w > 0 ? s_wsum[w - 1] : 0);
    if (e0 < E) s_off[e0] = base;
    if (e1 < E) s_off[e1] = base + p0;
    if (tid == 0) s_off[E] = s_wsum[LT_WARPS - 1];
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int e = tid; e <= E; e += LT_THREADS) offsets[e] = s_off[e];
        for (int e = tid; e < E; e += LT_THREADS) counts[e] = s_tot[e];
        const int Eloc = E / R;
        for (int r = tid; r <= R; r += LT_THREADS) rank_offsets[r] = s_off[r * Eloc];
        if (tid == 0 && (int64_t)s_off[E] > cap) set_status(status, MOE_STATUS_OVERFLOW);
    }

    // ---- phase 2c: slots of this CTA's tiles ----
    bool over = false;
    for (int tile = t0; tile < t1; ++tile) {
        if (!single) {
            for (int i = tid; i < LT_WARPS * E; i += LT_THREADS) whist[i] = 0;
            __syncthreads();
            rank_tile(topk_idx, npairs, E, tile, w, lane, whist, my_e, my_r);
            __syncthreads();
        }
        // per-warp counts -> exclusive prefix over warps; the tile total moves the base on
        for (int e = tid; e < E; e += LT_THREADS) {
            int run = 0;
#pragma unroll
            for (int ww = 0; ww < LT_WARPS; ++ww) {
                const int cnt = whist[ww * E + e];
                whist[ww * E + e] = (uint16_t)run;
                run += cnt;
            }
            s_all[e] = s_off[e] + s_base[e];  // first row of this tile's pairs of expert e
            s_base[e] += run;
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < LT_ITEMS; ++it) {
            const int p = tile * LT_TILE + (w * LT_ITEMS + it) * 32 + lane;
            if (p >= npairs) continue;
            const int e = my_e[it];
            int sl = -1;
            if (e >= 0) {
                sl = s_all[e] + whist[w * E + e] + my_r[it];
                if ((int64_t)sl >= cap) {
                    sl = -1;
                    over = true;
                }
            }
            slot_of[p] = sl;
            if (sl >= 0) row_src[sl] = p;
        }
        __syncthreads();
    }
    if (over) set_status(status, MOE_STATUS_OVERFLOW);

    // ---- padding rows (one warp per expert) and rows past the layout ----
    const int gw = blockIdx.x * LT_WARPS + w, nw = gridDim.x * LT_WARPS;
    for (int e = gw; e < E; e += nw) {
        const int64_t lo = (int64_t)s_off[e] + s_tot[e];
        int64_t hi = s_off[e + 1];
        if (hi > cap) hi = cap;
        for (int64_t r = lo + lane; r < hi; r += 32) row_src[r] = -1;
    }
    for (int64_t r = (int64_t)s_off[E] + (int64_t)blockIdx.x * LT_THREADS + tid; r < cap;
         r += (int64_t)gridDim.x * LT_THREADS)
        row_src[r] = -1;
}

// ------------------------------------------------------------------------------------------
// Cluster layout: up to LC_MAX_CTAS tiles of LC_TILE pairs, one CTA each, all
// in one thread-block cluster (E <= LC_THREADS).  Each CTA ranks its tile (as
// above) and stores its tile histogram into every CTA's shared memory
// (distributed shared memory); after one hardware cluster barrier each CTA
// has all tiles' counts locally: the per-expert totals and the counts of the
// tiles below it.  No global scratch, no atomics, no spin-wait.
// ------------------------------------------------------------------------------------------

constexpr int LC_WARPS = 16;
constexpr int LC_THREADS = LC_WARPS * 32;
constexpr int LC_ITEMS = 4;
constexpr int LC_TILE = LC_THREADS * LC_ITEMS;  // 2048 pairs per CTA
// 16 CTAs: above the portable cluster size of 8, allowed per function (the
// layout falls back to the other paths where the device refuses it).  In the
// DeepSeek-V3-shaped prefill step, 16 CTAs of 512 threads beat 8 CTAs of 1024.
constexpr int LC_MAX_CTAS = 16;

__global__ void __launch_bounds__(LC_THREADS)
    layout_cluster_kernel(const int32_t *__restrict__ topk_idx, int npairs, int E, int R, int P, int64_t cap,
                          int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                          int32_t *__restrict__ rank_offsets, int32_t *__restrict__ slot_of,
                          int32_t *__restrict__ row_src, int32_t *status) {
    extern __shared__ __align__(16) uint8_t lc_smem[];
    int *allh = reinterpret_cast<int *>(lc_smem);              // [LC_MAX_CTAS][E] every tile's counts, pushed by its CTA
    int *thist = allh + LC_MAX_CTAS * E;                        // [E] this tile's counts
    int *s_tot = thist + E;                                     // [E] totals
    int *s_base = s_tot + E;                                    // [E] first row of this tile's pairs, per expert
    int *s_off = s_base + E;                                    // [E + 1] padded offsets
    int *s_lbase = s_off + E + 1;                               // [E] first position of expert e in the tile's sorted order
    int *loc_p = s_lbase + E;                                   // [LC_TILE] the tile's pairs sorted by (expert, pair)
    int *loc_s = loc_p + LC_TILE;                               // [LC_TILE] their slots
    // [LC_WARPS][E + 2]: the padded row stride moves each warp's row by one bank
    uint16_t *whist = reinterpret_cast<uint16_t *>(loc_s + LC_TILE + 3);
    const int WS = E + 2;
    __shared__ int s_wsum[LC_WARPS];
    __shared__ int s_lsum[LC_WARPS];

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int C = gridDim.x;
    const uint32_t me = cluster_ctarank();
    const int tile = blockIdx.x;
    for (int i = tid; i < LC_WARPS * WS; i += LC_THREADS) whist[i] = 0;
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    // ---- rank this CTA's pairs: warp w takes LC_ITEMS consecutive chunks of 32 ----
    const unsigned lt = lanemask_lt();
    int my_e[LC_ITEMS], my_r[LC_ITEMS];
    int ev[LC_ITEMS];
#pragma unroll
    for (int it = 0; it < LC_ITEMS; ++it) {
        const int p = tile * LC_TILE + (w * LC_ITEMS + it) * 32 + lane;
        ev[it] = p < npairs ? __ldcg(topk_idx + p) : -1;  // through L2: written by the previous kernel
    }
    bool bad = false;
#pragma unroll
    for (int it = 0; it < LC_ITEMS; ++it) {
        const int p = tile * LC_TILE + (w * LC_ITEMS + it) * 32 + lane;
        int e = ev[it];
        if (p < npairs && (e < 0 || e >= E)) {
            bad = true;
            e = -1;
        }
        const unsigned peers = expert_peers(e, expert_bits(E));
        const int before = e >= 0 ? (int)whist[w * WS + e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) whist[w * WS + e] = (uint16_t)(before + __popc(peers));
        __syncwarp();
        my_e[it] = e;
        my_r[it] = before + __popc(peers & lt);
    }
    if (bad) set_status(status, MOE_STATUS_BAD_INDEX);
    __syncthreads();
    // per-warp counts -> exclusive prefix over warps, and the tile's total per
    // expert: tpe consecutive lanes share an expert, each summing LC_WARPS / tpe
    // warps, then an exclusive scan across those lanes (shuffles)
    int tpe = 1;
    while (tpe < 32 && tpe < LC_WARPS && tpe * 2 * E <= LC_THREADS) tpe *= 2;
    {
        const int wpt = LC_WARPS / tpe, sub = lane & (tpe - 1), epw = 32 / tpe;
        const int w0 = sub * wpt;
        for (int e0 = w * epw; e0 < E; e0 += LC_WARPS * epw) {  // warp-uniform trip count
            const int e = e0 + lane / tpe;
            const bool ok = e < E;
            int part = 0;
            if (ok)
                for (int ww = w0; ww < w0 + wpt; ++ww) part += whist[ww * WS + e];
            int incl = part;  // inclusive scan over the tpe lanes of this expert
            for (int off = 1; off < tpe; off <<= 1) {
                const int o = __shfl_up_sync(FULL, incl, off, tpe);
                if (sub >= off) incl += o;
            }
            if (ok) {
                int run = incl - part;
                for (int ww = w0; ww < w0 + wpt; ++ww) {
                    const int c = whist[ww * WS + e];
                    whist[ww * WS + e] = (uint16_t)run;
                    run += c;
                }
                if (sub == tpe - 1) thist[e] = incl;
            }
        }
    }
    __syncthreads();
    // push this tile's counts into row `me` of every CTA's allh (stores into the
    // cluster's distributed shared memory), then one cluster barrier: after it
    // every CTA holds all tiles' counts locally, and no CTA touches another's
    // shared memory again, so none has to wait for the others before exiting
    const uint32_t ah = smem_addr(allh) + 4u * me * (uint32_t)E;
    for (int idx = tid; idx < C * E; idx += LC_THREADS) {
        const int c = idx / E, e = idx - c * E;
        st_cluster_s32(cluster_map(ah + 4u * e, (uint32_t)c), thist[e]);
    }
    cluster_arrive();
    cluster_wait();

    // ---- totals and the count of the tiles below this one ----
    for (int e = tid; e < E; e += LC_THREADS) {
        int all = 0, below = 0;
        for (int c = 0; c < C; ++c) {
            const int v = allh[c * E + e];
            all += v;
            below += (uint32_t)c < me ? v : 0;
        }
        s_tot[e] = all;
        s_base[e] = below;
    }
    __syncthreads();

    // ---- exclusive scans over experts (one expert per thread): the padded
    // totals give the offsets, this tile's counts give its local sorted order ----
    const int pc = tid < E ? pad_count(s_tot[tid], P) : 0;
    const int lc = tid < E ? thist[tid] : 0;
    int incl = pc, lincl = lc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(FULL, incl, off);
        const int lo = __shfl_up_sync(FULL, lincl, off);
        if (lane >= off) {
            incl += o;
            lincl += lo;
        }
    }
    if (lane == 31) {
        s_wsum[w] = incl;
        s_lsum[w] = lincl;
    }
    __syncthreads();
    if (w == 0) {
        int v = lane < LC_WARPS ? s_wsum[lane] : 0;
        int lv = lane < LC_WARPS ? s_lsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(FULL, v, off);
            const int lo = __shfl_up_sync(FULL, lv, off);
            if (lane >= off) {
                v += o;
                lv += lo;
            }
        }
        if (lane < LC_WARPS) {
            s_wsum[lane] = v;  // inclusive over warps
            s_lsum[lane] = lv;
        }
    }
    __syncthreads();
    if (tid < E) {
        const int off = incl - pc + (w > 0 ? s_wsum[w - 1] : 0);
        s_off[tid] = off;
        s_base[tid] += off;
        s_lbase[tid] = lincl - lc + (w > 0 ? s_lsum[w - 1] : 0);
    }
    if (tid == 0) s_off[E] = s_wsum[LC_WARPS - 1];
    const int nsorted = s_lsum[LC_WARPS - 1];  // this tile's pairs with a valid expert
    __syncthreads();
    if (me == 0) {
        for (int e = tid; e <= E; e += LC_THREADS) offsets[e] = s_off[e];
        for (int e = tid; e < E; e += LC_THREADS) counts[e] = s_tot[e];
        const int Eloc = E / R;
        for (int r = tid; r <= R; r += LC_THREADS) rank_offsets[r] = s_off[r * Eloc];
        if (tid == 0 && (int64_t)s_off[E] > cap) set_status(status, MOE_STATUS_OVERFLOW);
    }

    // ---- slots ----
    bool over = false;
#pragma unroll
    for (int it = 0; it < LC_ITEMS; ++it) {
        const int p = tile * LC_TILE + (w * LC_ITEMS + it) * 32 + lane;
        if (p >= npairs) continue;
        const int e = my_e[it];
        int sl = -1;
        if (e >= 0) {
            const int within = whist[w * WS + e] + my_r[it];  // earlier pairs of e in this tile
            sl = s_base[e] + within;
            if ((int64_t)sl >= cap) {
                sl = -1;
                over = true;
            }
            const int lp = s_lbase[e] + within;
            loc_p[lp] = p;
            loc_s[lp] = sl;
        }
        slot_of[p] = sl;
    }
    if (over) set_status(status, MOE_STATUS_OVERFLOW);
    __syncthreads();
    // row_src in slot order: consecutive threads write the consecutive rows of
    // each expert's run, so a warp's stores share sectors
    for (int j = tid; j < nsorted; j += LC_THREADS) {
        const int sl = loc_s[j];
        if (sl >= 0) row_src[sl] = loc_p[j];
    }

    // ---- padding rows (one warp per expert) and rows past the layout ----
    const int gw = tile * LC_WARPS + w, nw = C * LC_WARPS;
    for (int e = gw; e < E; e += nw) {
        const int64_t lo = (int64_t)s_off[e] + s_tot[e];
        int64_t hi = s_off[e + 1];
        if (hi > cap) hi = cap;
        for (int64_t r = lo + lane; r < hi; r += 32) row_src[r] = -1;
    }
    for (int64_t r = (int64_t)s_off[E] + (int64_t)tile * LC_THREADS + tid; r < cap; r += (int64_t)C * LC_THREADS)
        row_src[r] = -1;
}

static cudaError_t launch_layout_cluster(const int32_t *topk_idx, int npairs, int E, int R, int P, int64_t cap,
                                         int32_t *counts, int32_t *offsets, int32_t *rank_offsets,
                                         int32_t *slot_of, int32_t *row_src, int32_t *status, cudaStream_t st,
                                         bool *launched, bool dry = false) {
    *launched = false;
    const int C = (npairs + LC_TILE - 1) / LC_TILE;
    if (C < 1 || C > LC_MAX_CTAS || E > LC_THREADS) return cudaSuccess;  // not launched
    // ints: allh [LC_MAX_CTAS][E], thist, s_tot, s_base [E] each, s_off [E + 1], s_lbase [E],
    // loc_p, loc_s [LC_TILE] each, 3 of padding; then whist
    const size_t smem = (size_t)((LC_MAX_CTAS + 5) * E + 2 * LC_TILE + 4) * sizeof(int) +
                        (size_t)LC_WARPS * (E + 2) * sizeof(uint16_t);
    static KernelSlots<decltype(&layout_cluster_kernel)> slots;
    int sms = 0, per_sm = 0;
    cudaError_t e = slots.prepare(&layout_cluster_kernel, LC_THREADS, smem, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaSuccess;
    static PerDeviceFlag pdl_ok, cluster_ok;
    if (!cluster_ok.on()) return cudaSuccess;
    if (dry) {
        *launched = true;
        return cudaSuccess;
    }
    if (C > 8) {  // clusters above the portable size must be allowed per function
        e = cudaFuncSetAttribute(layout_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            cluster_ok.disable();
            return cudaSuccess;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C);
    cfg.blockDim = dim3(LC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_ok.on() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, layout_cluster_kernel, topk_idx, npairs, E, R, P, cap, counts, offsets,
                           rank_offsets, slot_of, row_src, status);
    if (e != cudaSuccess && cfg.numAttrs == 2) {
        (void)cudaGetLastError();  // the pair was refused: launch without PDL on this device from now on
        pdl_ok.disable();
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, layout_cluster_kernel, topk_idx, npairs, E, R, P, cap, counts, offsets,
                               rank_offsets, slot_of, row_src, status);
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();  // no cluster launch on this device: the other paths from now on
        cluster_ok.disable();
        return cudaSuccess;
    }
    *launched = true;
    return cudaSuccess;
}

static cudaError_t launch_layout_fused(const int32_t *topk_idx, int npairs, int E, int R, int P, int64_t cap, int T,
                                       int32_t *hist, LayoutHeader *hdr, int32_t *counts, int32_t *offsets,
                                       int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src, int32_t *status,
                                       cudaStream_t st, bool *launched, bool dry = false) {
    *launched = false;
    const size_t smem = (size_t)((LT_WARPS * E * 2 + 15) & ~15) + 2 * 1024 * sizeof(int);
    static KernelSlots<decltype(&layout_fused_kernel)> slots;
    int sms = 0, per_sm = 0;
    cudaError_t e = slots.prepare(&layout_fused_kernel, LT_THREADS, smem, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    long long grid = (long long)sms * per_sm;  // all CTAs must be co-resident
    if (grid > T) grid = T;
    if (grid < 1 || (long long)T * E > LF_MAX_HIST) return cudaSuccess;  // not launched: use two kernels
    if (dry) {
        *launched = true;
        return cudaSuccess;
    }
    // Cooperative (all CTAs co-resident, for the grid barrier) and, where the
    // driver accepts the pair, programmatic serialisation too (see pdl_wait).
    static PerDeviceFlag pdl_ok;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(LT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_ok.on() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, layout_fused_kernel, topk_idx, npairs, E, R, P, cap, T, hist, hdr, counts,
                           offsets, rank_offsets, slot_of, row_src, status);
    if (e != cudaSuccess && cfg.numAttrs == 2) {
        (void)cudaGetLastError();  // the pair was refused: launch cooperative only on this device from now on
        pdl_ok.disable();
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, layout_fused_kernel, topk_idx, npairs, E, R, P, cap, T, hist, hdr, counts,
                               offsets, rank_offsets, slot_of, row_src, status);
    }
    if (e == cudaSuccess) *launched = true;
    return e;
}

int layout_kernel_count(int S, int E, int K) {
    const int npairs = S * K;
    bool one = false;
    if (launch_layout_cluster(nullptr, npairs, E, 1, 0, 0, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                              nullptr, &one, true) != cudaSuccess)
        return -1;
    if (one) return 1;
    if (launch_layout_fused(nullptr, npairs, E, 1, 0, 0, layout_tiles(npairs), nullptr, nullptr, nullptr, nullptr,
                            nullptr, nullptr, nullptr, nullptr, nullptr, &one, true) != cudaSuccess)
        return -1;
    return one ? 1 : 2;
}

cudaError_t launch_layout(const int32_t *topk_idx, int S, int E, int K, int R, int P,
                          int32_t *counts, int32_t *offsets, int32_t *rank_offsets,
                          int32_t *slot_of, int32_t *row_src, int64_t cap, void *workspace,
                          int32_t *status, cudaStream_t st) {
    const int npairs = S * K;
    const int T = layout_tiles(npairs);
    auto *hdr = reinterpret_cast<LayoutHeader *>(workspace);
    auto *hist = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(workspace) + LT_HEADER);
    bool launched = false;
    cudaError_t ce = launch_layout_cluster(topk_idx, npairs, E, R, P, cap, counts, offsets, rank_offsets, slot_of,
                                           row_src, status, st, &launched);
    if (ce != cudaSuccess) return ce;
    if (launched) return cudaSuccess;
    cudaError_t fe = launch_layout_fused(topk_idx, npairs, E, R, P, cap, T, hist, hdr, counts, offsets,
                                         rank_offsets, slot_of, row_src, status, st, &launched);
    if (fe != cudaSuccess) return fe;
    if (launched) return cudaSuccess;
    const size_t smem = (size_t)LT_WARPS * E * sizeof(uint16_t);
    static KernelSlots<decltype(&layout_hist_kernel)> hist_slots;
    static KernelSlots<decltype(&layout_slots_kernel)> slot_slots;
    int n_sms = 0, per_sm = 0;
    cudaError_t err = hist_slots.prepare(&layout_hist_kernel, LT_THREADS, smem, &n_sms, &per_sm);
    if (err != cudaSuccess) return err;
    err = slot_slots.prepare(&layout_slots_kernel, LT_THREADS, smem, &n_sms, &per_sm);
    if (err != cudaSuccess) return err;
    err = launch_pdl(layout_hist_kernel, dim3(T), dim3(LT_THREADS), smem, st, topk_idx, npairs,
                                 E, R, P, cap, hist, hdr, counts, offsets, rank_offsets, status);
    if (err != cudaSuccess) return err;
    return launch_pdl(layout_slots_kernel, dim3(T), dim3(LT_THREADS), smem, st, topk_idx, npairs, E,
                      (const int32_t *)hist, (const int32_t *)counts, (const int32_t *)offsets, cap, slot_of,
                      row_src, status);
}

}  // namespace moe
