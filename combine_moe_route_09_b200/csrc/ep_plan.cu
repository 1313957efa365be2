// Expert-parallel receive plan (host only): where each source rank's rows of
// each expert land in the owning rank's receive buffer.
//
// "Efficient and portable mixture-of-experts communication", Portable
// Kernels: experts are split over the ranks in blocks of E/W, and a fixed
// region per (source rank, local expert) gives every sender a unique place to
// write; Dispatch: the rows of one expert are contiguous at the receiver,
// whichever rank sent them.  "MoonEP developer guide", core API example:
// Buffer(S, H, K, E, num_ep_ranks), tokens_per_expert, cu_seqlens and
// token_padding.
//
// With the per-rank counts C[s][e] exchanged (an all-gather), every rank
// derives the same plan without further communication:
//   tot[e]   = sum_s C[s][e];  pc[e] = tot[e] rounded up to a multiple of P
//   expert_offsets[e] = sum_{e' < e} pc[e']  (all ranks' receive buffers one
//                       after the other, rank-major: the single-GPU layout)
//   recv_rows[d]      = sum of pc[e] over rank d's experts
//   recv_offsets[d][s][j] = (expert_offsets[e] - expert_offsets[d*Eloc])
//                           + sum_{s' < s} C[s'][e],   e = d*Eloc + j
// so that source rank s's rows of expert e occupy
//   [recv_offsets[d][s][j], + C[s][e]) in rank d's receive buffer,
// ordered within an expert by (source rank, source token): with tokens split
// over ranks in contiguous blocks this is ascending global token order, the
// single-GPU layout's order.
#include <stddef.h>
#include <stdint.h>

#include "moe_route.h"

extern "C" int moe_ep_plan(const int32_t *counts, int W, int E, int token_padding, int32_t *expert_offsets,
                           int32_t *recv_offsets, int32_t *recv_rows) {
    if (!counts || !expert_offsets || !recv_offsets || !recv_rows) return MOE_ERR_INVALID_ARG;
    if (W < 1 || E < 1 || E > MOE_MAX_EXPERTS || E % W != 0 || token_padding < 0) return MOE_ERR_INVALID_ARG;
    const int Eloc = E / W;
    // totals per expert, padded, and the exclusive scan over experts
    int64_t run = 0;
    for (int e = 0; e < E; ++e) {
        int64_t tot = 0;
        for (int s = 0; s < W; ++s) {
            const int32_t c = counts[(size_t)s * E + e];
            if (c < 0) return MOE_ERR_INVALID_ARG;
            tot += c;
        }
        const int64_t pc = token_padding > 0 ? (tot + token_padding - 1) / token_padding * token_padding : tot;
        expert_offsets[e] = (int32_t)run;
        run += pc;
        if (run >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
    }
    expert_offsets[E] = (int32_t)run;
    for (int d = 0; d < W; ++d) {
        const int32_t base = expert_offsets[d * Eloc];
        recv_rows[d] = expert_offsets[(d + 1) * Eloc] - base;
        for (int j = 0; j < Eloc; ++j) {
            const int e = d * Eloc + j;
            int32_t at = expert_offsets[e] - base;
            for (int s = 0; s < W; ++s) {
                recv_offsets[((size_t)d * W + s) * Eloc + j] = at;
                at += counts[(size_t)s * E + e];
            }
        }
    }
    return MOE_OK;
}
