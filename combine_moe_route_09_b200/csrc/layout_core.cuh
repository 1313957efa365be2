// Pieces of the dispatch layout shared by the layout kernels (layout.cu) and
// the fused route + dispatch kernel: the padded count, the peer masks that
// rank a warp's pairs by expert without atomics, the scratch header and the
// bounded grid barrier of a cooperative launch.
#pragma once

#include "common.cuh"
#include "tma.cuh"

namespace moe {

// The first bytes of the layout workspace (zero before the first call; every
// completed call leaves them ready for the next).
struct LayoutHeader {
    unsigned int ticket;   // two-kernel path: arrival ticket, reset by the last CTA
    unsigned int count;    // grid barrier: arrivals, reset by the last arriver
    unsigned int gen;      // grid barrier: generation (only ever incremented)
};

// Rows of an expert with c pairs: c rounded up to a multiple of P (P = 0: c).
__device__ __forceinline__ int pad_count(int c, int P) { return P > 0 ? ((c + P - 1) / P) * P : c; }

// Lanes of the warp holding the same expert id as this lane (e = -1: none).
// One ballot per bit of the id (ids below 2^nbits) plus one for validity: a
// fixed, short sequence, where __match_any_sync takes longer the more
// distinct values the warp holds.
__device__ __forceinline__ unsigned expert_peers(int e, int nbits) {
    unsigned peers = __ballot_sync(FULL, e >= 0);
    if (e < 0) peers = ~peers;
    for (int b = 0; b < nbits; ++b) {
        const bool bit = (e >> b) & 1;
        const unsigned m = __ballot_sync(FULL, bit);
        peers &= bit ? m : ~m;
    }
    return peers;
}

// Bits that cover every expert id below E.
__device__ __forceinline__ int expert_bits(int E) { return E > 1 ? 32 - __clz(E - 1) : 0; }

// Grid-wide barrier for a cooperative launch (all CTAs co-resident), run by
// ONE thread per CTA after the CTA's own writes that must be visible (the
// caller synchronises its threads around it).  Sense reversal: read the
// generation, arrive; the last arriver resets the count and bumps the
// generation; the others wait (bounded) for the bump.  False on timeout
// (MOE_STATUS_TIMEOUT is then set).
__device__ __forceinline__ bool grid_arrive_wait(LayoutHeader *hdr, int32_t *status) {
    bool ok = true;
    const unsigned gen = *(volatile unsigned *)&hdr->gen;
    __threadfence();
    const unsigned prev = atomicAdd(&hdr->count, 1u);
    if (prev == gridDim.x - 1) {
        *(volatile unsigned *)&hdr->count = 0u;
        __threadfence();
        atomicExch(&hdr->gen, gen + 1u);
    } else {
        ok = wait_changed_for(&hdr->gen, gen, status, MOE_WAIT_NS);
    }
    __threadfence();
    return ok;
}

}  // namespace moe
