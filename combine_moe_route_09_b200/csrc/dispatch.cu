// Dispatch: scatter each token row into the K rows its (token, k) pairs were
// given, optionally quantised to FP8 e4m3 with one fp32 scale per 128 channels.
//
// "Efficient and portable mixture-of-experts communication", Dispatch: tokens
// and their block scaling factors are packed and laid out contiguously per
// expert for the grouped GEMM.  "DeepSeek AI releases DeepEP", Technical
// overview: the dispatch may carry FP8.
//
// Both kernels are persistent over work items = (token, column chunk), each
// CTA taking a contiguous, balanced share, and move rows with TMA bulk copies (cp.async.bulk; no tensor maps, no
// multicast): each row chunk is read from HBM once and written K times.
//
//  dispatch_copy_kernel (no quantisation, bf16 or fp32): one warp per CTA,
//    a contiguous share of the items.  A ring of shared-memory stages; lane 0
//    bulk-loads item i+STAGES-1 while the K bulk stores of item i go out
//    straight from its stage (lane k stores copy k; the token's slots are
//    loaded one token ahead).  A stage is reloaded only after its stores have
//    finished reading it (cp.async.bulk.wait_group.read).
//
//  dispatch_fp8_kernel: each CTA again takes a contiguous share, so
//    consecutive items mostly belong to one token.  A producer warp
//    bulk-loads input chunks into a ring of stages and puts the token's slots
//    (loaded one token ahead) in each stage's header; 8 consumer warps
//    quantise: each thread owns 16 channels, the 8 threads of a 128-channel
//    block reduce amax with xor-shuffles, s = amax / 448 (IEEE division) and
//    q = e4m3(x / s) with the quotient correctly rounded (Markstein's
//    correction of x * RN(1/s); plain IEEE division for s < 2^-90) and
//    cvt.rn.satfinite.e4m3x2.  With at least DQ_BULK_MIN_ITEMS_PER_SM items
//    per SM the quantised item (codes, then its block scales) is staged in
//    one of DQ_OUT_BUFS shared-memory buffers, and after a named barrier one
//    thread sends the K copies as TMA bulk stores (one per copy for the
//    codes, one for the scales when the segment is whole 16-byte units, else
//    the blocks' lead threads store the scales): whole-item bulk stores write
//    the scattered destination rows faster.  With fewer items (decode sizes)
//    each thread stores its codes K times from registers, which is faster
//    when the staging cannot be amortised.
#include "common.cuh"
#include "kernels.cuh"
#include "fp8_core.cuh"
#include "tma.cuh"

namespace moe {

// ------------------------------------------------------------------------------------------
// plain copy
// ------------------------------------------------------------------------------------------

// A 12-stage ring of 2 KB chunks (24 KB per CTA, as the earlier 6 x 4 KB).  In
// the graph-replayed step, three interleaved process pairs: 16384 x 2048 rows
// 253.6 -> 252.3 us, 4096 x 768 40.9 -> 40.6 us, 1024 x 768 19.09 -> 18.85 us;
// 8 x 4 KB and 4 x 4 KB landed in between, 6 x 2 KB was slower (260.6 us).
constexpr int DC_STAGES = 12;
constexpr int DC_CHUNK = 2048;

struct CopyArgs {
    const uint8_t *x;
    const int32_t *slot_of;
    uint8_t *xd;
    int32_t *status;
    int64_t cap;
    int S, K;
    int row_bytes, chunk, nchunks;
};

// Items [first, last) of this CTA: a contiguous, balanced share of n items.
__device__ __forceinline__ void cta_range(long long n, long long &first, long long &last) {
    first = n * blockIdx.x / gridDim.x;
    last = n * (blockIdx.x + 1) / gridDim.x;
}

__global__ void __launch_bounds__(32) dispatch_copy_kernel(const CopyArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + DC_STAGES * a.chunk);
    const uint32_t smem0 = smem_addr(smem), bar0 = smem_addr(bars);
    const int lane = threadIdx.x;
    if (lane == 0) {
        for (int s = 0; s < DC_STAGES; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    pdl_wait();
    pdl_trigger();

    long long first, last;
    cta_range((long long)a.S * a.nchunks, first, last);
    const int n = (int)(last - first);
    // Loads run DC_STAGES - 1 items ahead of the stores; each side walks its
    // (token, chunk) pair incrementally.
    int lt = (int)(first / a.nchunks), lc = (int)(first - (long long)lt * a.nchunks);
    auto load = [&](int j) {  // lane 0 only; j = next item to load, in order
        const int off = lc * a.chunk;
        const uint32_t bytes = (uint32_t)min(a.chunk, a.row_bytes - off);
        const uint32_t bar = bar0 + 8u * (j % DC_STAGES);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(smem0 + (uint32_t)((j % DC_STAGES) * a.chunk), a.x + (size_t)lt * a.row_bytes + off, bytes, bar);
    };
    auto advance = [&]() {
        if (++lc == a.nchunks) {
            lc = 0;
            ++lt;
        }
    };
    for (int j = 0; j < DC_STAGES - 1 && j < n; ++j) {
        if (lane == 0) load(j);
        advance();
    }
    int issued = min(DC_STAGES - 1, n);  // loads issued (lane 0's count, kept uniform)

    // Lane k holds the current token's slot k; the next token's is loaded ahead.
    int t_cur = -1, cur = -1, nxt = -1;
    if (n > 0 && lane < a.K) nxt = __ldg(a.slot_of + (size_t)(first / a.nchunks) * a.K + lane);
    bool ok = true;
    int i = 0;
    int t = (int)(first / a.nchunks), c = (int)(first - (long long)t * a.nchunks);
    for (; i < n; ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
        if (t != t_cur) {
            t_cur = t;
            cur = nxt;
            if ((int64_t)cur >= a.cap) {
                set_status(a.status, MOE_STATUS_BAD_SLOT);
                cur = -1;
            }
            if (lane < a.K && (long long)(t + 1) * a.nchunks < last)
                nxt = __ldg(a.slot_of + (size_t)(t + 1) * a.K + lane);
        }
        const int off = c * a.chunk;
        const uint32_t bytes = (uint32_t)min(a.chunk, a.row_bytes - off);
        const int s = i % DC_STAGES;
        ok = __all_sync(FULL, mbar_wait(bar0 + 8u * s, (i / DC_STAGES) & 1, a.status));
        if (!ok) break;  // uniform: decided by __all_sync
        // every lane with a valid slot stores its copy straight from the stage
        if (cur >= 0) bulk_s2g(a.xd + (size_t)cur * a.row_bytes + off, smem0 + (uint32_t)(s * a.chunk), bytes);
        bulk_commit();
        const int j = i + DC_STAGES - 1;
        if (j < n) {
            // stage j % STAGES last held item i-1: its stores must have read it
            bulk_wait_read<1>();
            __syncwarp();
            if (lane == 0) load(j);
            advance();
            issued = j + 1;
        }
    }
    // After an early exit, loads i .. issued-1 may still be landing in shared
    // memory: wait for them (bounded) before the CTA's memory is released.
    if (!ok && lane == 0)
        for (int j = i; j < issued; ++j) mbar_wait(bar0 + 8u * (j % DC_STAGES), (j / DC_STAGES) & 1, a.status);
    bulk_wait_all();
}

// ------------------------------------------------------------------------------------------
// FP8 e4m3, 128-channel blocks
// ------------------------------------------------------------------------------------------

// 8 consumer warps take up to 64 blocks (8192 channels) per item -- a whole
// 7168-channel row -- through a 96 KB input ring (6 stages, two CTAs per SM).
// In the DeepSeek-V3-shaped prefill step (graph replays) this ran 175.1 us per
// step against 177.7 us for 4 warps with half rows in a 48 KB ring; a 64 KB
// ring gave 176.2 us and a 128 KB ring (one CTA per SM) 194.8 us.
constexpr int DQ_MAX_STAGES = 8;
constexpr int DQ_STAGE_BUDGET = 96 * 1024;                   // bytes of input ring per CTA
constexpr int DQ_CONSUMER_WARPS = 8;
constexpr int DQ_CONSUMERS = DQ_CONSUMER_WARPS * 32;
constexpr int DQ_THREADS = DQ_CONSUMERS + 32;
constexpr int DQ_UNIT = 16;                                  // channels of one thread unit
constexpr int DQ_UNITS = 2;                                  // units per thread and item
constexpr int DQ_SPAN = DQ_CONSUMERS * DQ_UNIT;              // channels between a thread's units
constexpr int DQ_MAX_BLOCKS = DQ_UNITS * DQ_SPAN / 128;      // 128-channel blocks per item
constexpr int DQ_HDR = 128;                                  // per-stage header: the token's K slots
constexpr int DQ_OUT_BUFS = 2;                 // bulk-store path: output staging buffers
constexpr int DQ_BULK_MIN_ITEMS_PER_SM = 16;                 // bulk-store path from this many items per SM

struct Fp8Args {
    const uint8_t *x;
    const int32_t *slot_of;
    uint8_t *xd;
    float *xs;
    int32_t *status;
    int64_t cap;
    int S, H, K;
    int esz;         // input element bytes (2 or 4)
    int bpc;         // 128-channel blocks per item (the last item of a row may hold fewer)
    int nchunks;     // items per token
    int stage;       // bytes per stage: header + bpc * 128 * esz
    int stages;      // stages in the ring (<= DQ_MAX_STAGES)
    int obuf;        // bulk-store path: bytes per output staging buffer (codes, then scales)
    int scale_bulk;  // bulk-store path: the item's scale segment is also one bulk store per copy
};

// KT: K known at compile time (0 = runtime K).  BULK: the K copies of an item
// leave through TMA bulk stores from a shared-memory staging buffer (one
// elected thread issues them) instead of per-thread 16-byte stores.
template <bool IN_F32, int KT, bool BULK>
__global__ void __launch_bounds__(DQ_THREADS) dispatch_fp8_kernel(const Fp8Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    // layout: [stages][header (K slots) | bpc*128*esz input bytes]
    //         | BULK: [DQ_OUT_BUFS][bpc*128 codes | bpc*4 scales, padded to 16] | barriers
    const int NS = a.stages;
    const int K = KT > 0 ? KT : a.K;
    const uint32_t smem0 = smem_addr(smem);
    const uint32_t obuf0 = smem0 + (uint32_t)(NS * a.stage);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + NS * a.stage + (BULK ? DQ_OUT_BUFS * a.obuf : 0));
    const uint32_t bar0 = smem_addr(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (DQ_MAX_STAGES + s); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), DQ_CONSUMER_WARPS);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    long long first, last;
    cta_range((long long)a.S * a.nchunks, first, last);
    const int row_bytes = a.H * a.esz;
    const int chunk_bytes = a.bpc * 128 * a.esz;
    const int nb = a.H >> 7;
    if (warp == DQ_CONSUMER_WARPS) {
        // ------------------------------- producer -------------------------------
        // The token's slots are loaded one token ahead (lane k holds slot k).
        int t_cur = -1;
        int nxt = -1;
        const int t_first = (int)(first / a.nchunks);
        if (first < last && lane < K) nxt = __ldg(a.slot_of + (size_t)t_first * K + lane);
        int cur = -1;
        int i = 0;
        bool ok = true;
        int t = t_first, c = (int)(first - (long long)t_first * a.nchunks);
        for (long long item = first; item < last && ok; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
            const int s = i % NS;
            if (t != t_cur) {
                t_cur = t;
                cur = nxt;
                if ((int64_t)cur >= a.cap) {
                    set_status(a.status, MOE_STATUS_BAD_SLOT);
                    cur = -1;
                }
                const int tn = t + 1;
                if (lane < K && (long long)tn * a.nchunks < last) nxt = __ldg(a.slot_of + (size_t)tn * K + lane);
            }
            if (i >= NS)
                ok = __all_sync(FULL, mbar_wait(empty_bar(s), ((i / NS) - 1) & 1, a.status));
            if (!ok) break;
            const int off = c * chunk_bytes;
            const uint32_t bytes = (uint32_t)min(chunk_bytes, row_bytes - off);
            const uint32_t st = smem0 + (uint32_t)(s * a.stage);
            if (lane < K) asm volatile("st.shared.s32 [%0], %1;" ::"r"(st + 4u * lane), "r"(cur) : "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(full_bar(s), bytes);
                bulk_g2s(st + DQ_HDR, a.x + (size_t)t * row_bytes + off, bytes, full_bar(s));
            }
        }
        if (lane == 0) {
            for (int j = i - NS; j < i; ++j)
                if (j >= 0) mbar_wait(full_bar(j % NS), (j / NS) & 1, a.status);
        }
        return;
    }

    // ------------------------------- consumers -------------------------------
    // Thread tid owns two 16-channel units of the item, channels
    // [16 tid + 2048 u, +16) for u = 0, 1 (two independent chains); the 8
    // threads of a 128-channel block reduce its amax.  BULK: the codes and the
    // blocks' scales go to a staging buffer and leave as bulk stores; otherwise
    // one 16-byte store per unit and copy (a warp writes 512 contiguous bytes
    // per copy) and the block's lead thread stores the scale.
    int t = (int)(first / a.nchunks), c = (int)(first - (long long)t * a.nchunks);
    int i = 0;
    for (long long item = first; item < last; ++item, ++i, (++c == a.nchunks ? (c = 0, ++t) : 0)) {
        const int s = i % NS;
        if constexpr (BULK) {
            // All 128 consumers leave together on a timeout (the staging buffer and
            // the barriers below are shared); the issuing thread first lets the
            // stores that last read this item's staging buffer finish reading it.
            const bool got = mbar_wait(full_bar(s), (i / NS) & 1, a.status);
            if (tid == 0) bulk_wait_read<DQ_OUT_BUFS - 1>();
            if (!named_bar_and(1, DQ_CONSUMERS, got)) break;
        } else {
            if (!__all_sync(FULL, mbar_wait(full_bar(s), (i / NS) & 1, a.status))) break;
        }
        const int col0 = c * a.bpc * 128;              // first channel of the item
        const int nch = min(a.bpc * 128, a.H - col0);  // channels in this item
        const uint32_t st = smem0 + (uint32_t)(s * a.stage);
        float f[DQ_UNITS][16];
        bool active[DQ_UNITS];
#pragma unroll
        for (int u = 0; u < DQ_UNITS; ++u) {
            const int ch = u * DQ_SPAN + tid * DQ_UNIT;
            active[u] = ch < nch;  // whole blocks: groups all-or-nothing
            if (active[u]) {
                const uint32_t src = st + DQ_HDR + (uint32_t)(ch * a.esz);
                if (IN_F32) {
#pragma unroll
                    for (int l = 0; l < 4; ++l) {
                        const U4 v = lds128(src + 16u * l);
                        f[u][4 * l + 0] = __uint_as_float(v.x);
                        f[u][4 * l + 1] = __uint_as_float(v.y);
                        f[u][4 * l + 2] = __uint_as_float(v.z);
                        f[u][4 * l + 3] = __uint_as_float(v.w);
                    }
                } else {
                    // Lanes sit 32 bytes apart, so a quarter-warp's first halves would
                    // share 16 banks; lanes 4-7 (mod 8) read their upper half first,
                    // which puts the eight 16-byte reads of each phase on distinct banks.
                    const uint32_t sw = (uint32_t)(lane >> 2) & 1u;
                    const U4 a0 = lds128(src + 16u * sw), a1 = lds128(src + 16u * (sw ^ 1u));
                    const U4 v2[2] = {sw ? a1 : a0, sw ? a0 : a1};
#pragma unroll
                    for (int l = 0; l < 2; ++l) {
                        const U4 &v = v2[l];
                        f[u][8 * l + 0] = bf16lo(v.x); f[u][8 * l + 1] = bf16hi(v.x);
                        f[u][8 * l + 2] = bf16lo(v.y); f[u][8 * l + 3] = bf16hi(v.y);
                        f[u][8 * l + 4] = bf16lo(v.z); f[u][8 * l + 5] = bf16hi(v.z);
                        f[u][8 * l + 6] = bf16lo(v.w); f[u][8 * l + 7] = bf16hi(v.w);
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) f[u][e] = 0.f;
            }
        }
        int myslot = -1;
        if (lane < K) asm volatile("ld.shared.s32 %0, [%1];" : "=r"(myslot) : "r"(st + 4u * lane) : "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));  // input stage no longer needed

        float scale[DQ_UNITS];
        U4 q[DQ_UNITS];
#pragma unroll
        for (int u = 0; u < DQ_UNITS; ++u) {
            float amax = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[u][e]));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 4));
            scale[u] = scale_of(amax);
            q[u] = quant16(f[u], scale[u]);
        }

        const bool lead = (lane & 7) == 0;
        if constexpr (BULK) {
            // stage the item (codes, then its scales), then one thread sends K copies
            const uint32_t ob = obuf0 + (uint32_t)((i % DQ_OUT_BUFS) * a.obuf);
            const int cbytes = a.bpc * 128;
#pragma unroll
            for (int u = 0; u < DQ_UNITS; ++u) {
                if (active[u]) {
                    const int ch = u * DQ_SPAN + tid * DQ_UNIT;
                    sts128(ob + (uint32_t)ch, q[u]);
                    if (lead) asm volatile("st.shared.f32 [%0], %1;" ::"r"(ob + (uint32_t)(cbytes + (ch >> 7) * 4)),
                                           "f"(scale[u]) : "memory");
                }
            }
            fence_proxy_async_smem();
            named_bar(2, DQ_CONSUMERS);
            const int nblk = nch >> 7;
            if (warp == 0) {
                for (int k = 0; k < K; ++k) {
                    const int sl = __shfl_sync(FULL, myslot, k);
                    if (lane == 0 && sl >= 0) {
                        bulk_s2g(a.xd + (size_t)sl * a.H + col0, ob, (uint32_t)nch);
                        if (a.scale_bulk)
                            bulk_s2g(a.xs + (size_t)sl * nb + (col0 >> 7), ob + (uint32_t)cbytes, (uint32_t)nblk * 4u);
                    }
                }
                if (lane == 0) bulk_commit();
            }
            if (!a.scale_bulk) {  // scales from registers, by each block's lead thread
                float *const scol = a.xs + ((col0 + tid * DQ_UNIT) >> 7);
                for (int k = 0; k < K; ++k) {
                    const int sl = __shfl_sync(FULL, myslot, k);
                    if (sl < 0 || !lead) continue;
#pragma unroll
                    for (int u = 0; u < DQ_UNITS; ++u)
                        if (active[u]) scol[(size_t)sl * nb + u * (DQ_SPAN >> 7)] = scale[u];
                }
            }
            continue;
        }
        uint8_t *const xcol = a.xd + col0 + tid * DQ_UNIT;
        float *const scol = a.xs + ((col0 + tid * DQ_UNIT) >> 7);
        constexpr int KU = KT > 0 ? KT : 1;
#pragma unroll(KU)
        for (int k = 0; k < K; ++k) {
            const int sl = __shfl_sync(FULL, myslot, k);
            if (sl < 0) continue;
            uint8_t *const row = xcol + (size_t)sl * a.H;
            float *const srow = scol + (size_t)sl * nb;
#pragma unroll
            for (int u = 0; u < DQ_UNITS; ++u) {
                if (active[u]) {
                    st_v4(row + u * DQ_SPAN, q[u]);
                    if (lead) srow[u * (DQ_SPAN >> 7)] = scale[u];
                }
            }
        }
    }
    if constexpr (BULK) {
        if (tid == 0) bulk_wait_all();  // this CTA's bulk stores are complete before it exits
    }
}

// ------------------------------------------------------------------------------------------

template <typename Kern>
static cudaError_t persistent_grid(KernelSlots<Kern> &slots, Kern kern, int threads, size_t smem,
                                   long long nitems, unsigned *grid) {
    int sms = 0, per_sm = 0;
    cudaError_t e = slots.prepare(kern, threads, smem, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    long long g = (long long)sms * per_sm;
    if (g > nitems) g = nitems;
    *grid = (unsigned)(g < 1 ? 1 : g);
    return cudaSuccess;
}

cudaError_t launch_dispatch(const void *x, int dtype, int S, int H, int K, const int32_t *slot_of,
                            int quant, void *xd, float *xs, int64_t cap, int32_t *status,
                            cudaStream_t st) {
    if (S == 0) return cudaSuccess;
    const int esz = dtype == MOE_DTYPE_F32 ? 4 : 2;
    const int row_bytes = H * esz;
    if (quant == MOE_QUANT_NONE) {
        CopyArgs a{reinterpret_cast<const uint8_t *>(x), slot_of, reinterpret_cast<uint8_t *>(xd), status,
                   cap, S, K, row_bytes, 0, 0};
        a.chunk = row_bytes < DC_CHUNK ? row_bytes : DC_CHUNK;
        a.nchunks = (row_bytes + a.chunk - 1) / a.chunk;
        const size_t smem = (size_t)DC_STAGES * a.chunk + DC_STAGES * 8;
        static KernelSlots<decltype(&dispatch_copy_kernel)> slots;
        unsigned grid = 1;
        cudaError_t e = persistent_grid(slots, &dispatch_copy_kernel, 32, smem, (long long)S * a.nchunks, &grid);
        if (e != cudaSuccess) return e;
        return launch_pdl(dispatch_copy_kernel, dim3(grid), dim3(32), smem, st, a);
    }
    Fp8Args a{reinterpret_cast<const uint8_t *>(x), slot_of, reinterpret_cast<uint8_t *>(xd), xs, status,
              cap, S, H, K, esz, 0, 0, 0, 0};
    // Split each row into the fewest items of at most DQ_MAX_BLOCKS blocks, as evenly as possible
    // (a multiple of 4 blocks where the row allows, so scale segments are whole 16-byte units).
    const int blocks = H / 128;
    const int n = (blocks + DQ_MAX_BLOCKS - 1) / DQ_MAX_BLOCKS;
    a.bpc = (blocks + n - 1) / n;
    if (blocks % 4 == 0) a.bpc = (a.bpc + 3) / 4 * 4;
    a.nchunks = (blocks + a.bpc - 1) / a.bpc;
    a.stage = DQ_HDR + a.bpc * 128 * esz;
    a.stages = DQ_STAGE_BUDGET / a.stage;
    if (a.stages > DQ_MAX_STAGES) a.stages = DQ_MAX_STAGES;
    if (a.stages < 3) a.stages = 3;
    a.obuf = a.bpc * 128 + (a.bpc * 4 + 15) / 16 * 16;
    a.scale_bulk = (blocks % 4 == 0 && a.bpc % 4 == 0 && (reinterpret_cast<uintptr_t>(xs) & 15) == 0) ? 1 : 0;
    const long long nitems = (long long)S * a.nchunks;
    // Bulk stores from a staging buffer pay off once each CTA has several items
    // to pipeline (prefill: 8192 items); with less than one item per CTA
    // (decode: 256) the staging and its barriers only add latency, and
    // per-thread stores are faster.
    int dev = 0, sm_count = 0;
    cudaError_t ae = cudaGetDevice(&dev);
    if (ae == cudaSuccess) ae = cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (ae != cudaSuccess) return ae;
    const bool bulk = nitems >= (long long)DQ_BULK_MIN_ITEMS_PER_SM * sm_count;
    const size_t smem = (size_t)a.stages * a.stage + (bulk ? (size_t)DQ_OUT_BUFS * a.obuf : 0) + 2 * DQ_MAX_STAGES * 8;
    auto go = [&](auto kern) -> cudaError_t {
        static KernelSlots<decltype(kern)> slots;
        unsigned grid = 1;
        cudaError_t e = persistent_grid(slots, kern, DQ_THREADS, smem, nitems, &grid);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, dim3(grid), dim3(DQ_THREADS), smem, st, a);
    };
    if (dtype == MOE_DTYPE_BF16) {
        if (bulk) return K == 8 ? go(&dispatch_fp8_kernel<false, 8, true>) : go(&dispatch_fp8_kernel<false, 0, true>);
        return K == 8 ? go(&dispatch_fp8_kernel<false, 8, false>) : go(&dispatch_fp8_kernel<false, 0, false>);
    }
    if (bulk) return K == 8 ? go(&dispatch_fp8_kernel<true, 8, true>) : go(&dispatch_fp8_kernel<true, 0, true>);
    return K == 8 ? go(&dispatch_fp8_kernel<true, 8, false>) : go(&dispatch_fp8_kernel<true, 0, false>);
}

}  // namespace moe
