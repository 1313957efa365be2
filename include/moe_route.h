/*
 * moe_route.h — C ABI of the B200 (sm_100a) MoE token dispatch / combine library.
 *
 * One forward pass of a Mixture-of-Experts layer's routing, on one GPU:
 *
 *   moe_route_topk            router top-K gating
 *   moe_dispatch_layout       per-expert histogram + prefix scan -> padded,
 *                             expert-contiguous (rank, local expert, slot) layout
 *   moe_dispatch              scatter token rows into that layout, optionally
 *                             quantised to FP8 e4m3 with one fp32 scale per
 *                             128-channel block
 *   moe_combine_dual_residual gather + top-K weighted sum back to token order,
 *                             fused with the FarSkip-Collective dual residual
 *
 * (moe_route_dispatch runs the first three as one call, in one kernel when the
 * batch fits) and around them: the backward of each step (moe_combine_dual_residual_backward,
 * moe_dispatch_backward, moe_route_topk_backward), the combine over FP8 expert
 * outputs (moe_combine_fp8_dual_residual), the routing weights in dispatched
 * order (moe_dispatch_route_weights), a sigmoid / selection-bias /
 * group-limited router (moe_route_sigmoid_grouped), an allocation-free layout
 * (moe_dispatch_layout_static) and host-side queries.
 *
 * Sources (page title, section):
 *   [pplx]    "Efficient and portable mixture-of-experts communication"
 *             (Perplexity, pplx-kernels): Introduction; Portable Kernels;
 *             Dispatch; Combine.
 *   [farskip] Instella-MoE-16B-A3B-SFT / FarSkip-Collective explainer: the dual
 *             residual stream and its four-line update.
 *   [deepep]  "DeepSeek AI releases DeepEP": Technical overview (FP8 dispatch).
 *   [moonep]  "MoonEP developer guide": core API example (Buffer(S, H, K, E,
 *             num_ep_ranks), dispatch -> tokens_per_expert / cu_seqlens / plan,
 *             combine(plan, ...)) and tuning parameters (token_padding = 128).
 *
 * Notation: S tokens (all R logical ranks together), H hidden size, E experts,
 * K experts per token, R logical expert-parallel ranks (experts split into R
 * contiguous blocks of E/R), P = token_padding (0 = none),
 * cap = rows of the dispatched buffer.  cap = S*K + E*max(P-1, 0) always fits.
 *
 * Conventions for every entry point
 *   - Every pointer except `stream` and those marked "host" is DEVICE memory
 *     that the caller allocated and owns.  The library allocates nothing and
 *     keeps no data between calls (only per-process launch settings: kernel
 *     attributes and occupancy answers, plus the fixed scratch array of
 *     moe_dispatch_layout_static), and it never synchronises with the host:
 *     all work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns once it is enqueued.
 *   - Arrays are dense row-major.  Activation buffers (x, xd, y, shared_out,
 *     residual, outputs) must be 16-byte aligned and their rows a multiple of
 *     16 bytes (H % 8 == 0 for bf16, H % 4 == 0 for f32, H % 128 == 0 for FP8).
 *     int32 / fp32 arrays must be 4-byte aligned.
 *   - Return value: MOE_OK, or MOE_ERR_INVALID_ARG when an argument fails the
 *     host-side checks stated for the call (nothing is enqueued then), or
 *     MOE_ERR_CUDA when a launch failed (cudaGetLastError() holds the cause).
 *   - Problems that only the data reveals (an expert id out of range, a slot
 *     outside [0, cap), a layout larger than cap) never fault: the offending
 *     element is skipped and a MOE_STATUS_* bit is OR-ed into *status, a
 *     device int32 the caller zeroes and reads whenever it likes.  `status`
 *     may be NULL, in which case such problems are skipped silently.
 *   - Every wait inside a kernel (pipeline barriers between the copy engine
 *     and the compute threads) is bounded in time; one that expires sets
 *     MOE_STATUS_TIMEOUT and the kernel returns instead of hanging.
 *   - Preconditions that are not checked: finite logits and activations.
 */
#ifndef MOE_ROUTE_H
#define MOE_ROUTE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG 1
#define MOE_ERR_CUDA 2
#define MOE_ERR_SCRATCH_TOO_SMALL 3 /* sizes need more scratch than moe_dispatch_layout_static has */

/* element types of activation buffers */
#define MOE_DTYPE_F32 0
#define MOE_DTYPE_BF16 1

/* dispatch quantisation */
#define MOE_QUANT_NONE 0
#define MOE_QUANT_FP8_E4M3_B128 1

/* device status bits (OR-ed into *status) */
#define MOE_STATUS_BAD_INDEX 1 /* an expert id outside [0, E); that pair was dropped */
#define MOE_STATUS_OVERFLOW 2  /* the padded layout needs more than cap rows */
#define MOE_STATUS_BAD_SLOT 4  /* a slot outside [0, cap) reached dispatch/combine; skipped */
#define MOE_STATUS_TIMEOUT 8   /* an internal pipeline wait exceeded its time bound; output incomplete */

#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 32

/*
 * Router top-K gating.  [pplx] Introduction: each token goes to the K experts
 * with the highest router scores; the expert outputs are summed with weights
 * taken from the router's probability distribution.
 *
 *   logits   [S, E] fp32 (device, read)
 *   topk_idx [S, K] int32 (device, written): the K largest logits of the row
 *            in descending order; equal logits -> lower expert id first;
 *            -0.0 and +0.0 are equal.
 *   topk_w   [S, K] fp32 (device, written): softmax over the K selected
 *            logits, w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0); this equals
 *            the full softmax over E renormalised over the chosen K.
 * Host checks: S >= 0, 1 <= E <= MOE_MAX_EXPERTS, 1 <= K <= min(E, MOE_MAX_TOPK),
 * non-NULL pointers when S > 0.
 */
MOE_API int moe_route_topk(const float *logits, int S, int E, int K, int32_t *topk_idx, float *topk_w,
                   void *stream);

/*
 * Self-test of the library's failure detection (no counterpart on the pages).
 * Runs one bounded wait that nothing will complete -- which = 0: an mbarrier
 * phase with no arrival; which = 1: a poll of *flag (device, 4 bytes, not
 * written by anyone while the test runs) -- with a limit of limit_ns
 * (1 .. 10^9 ns).  The wait runs out, sets MOE_STATUS_TIMEOUT in *status and
 * returns; the kernels of the library wait with these routines (200 ms limit).
 * Nothing traps or stays in flight.  flag may be NULL for which = 0.
 */
MOE_API int moe_selftest_wait_timeout(int which, unsigned long long limit_ns, int32_t *status, uint32_t *flag,
                                      void *stream);

/*
 * Number of kernels moe_dispatch_layout (and moe_dispatch_layout_static)
 * launches for these sizes on the current device: 1 (single-launch layouts:
 * a thread-block cluster for up to 32768 pairs and E <= 512, else a cooperative grid when
 * every CTA can scan the tile histograms) or 2 (histogram + slots).  For
 * sizing CUDA graphs and counting launches; no launch happens.  Returns -1 on
 * a CUDA error, 0 for invalid sizes.
 */
MOE_API int moe_dispatch_layout_kernels(int S, int E, int K);

/*
 * Routing weights in dispatched order (MoonEP developer guide, core API
 * example: the dispatch returns each expert's rows together with their routing
 * weights, which the combine consumes).
 *   topk_w         [S, K] fp32, from moe_route_topk / moe_route_sigmoid_grouped
 *   row_src        [cap] int32, from moe_dispatch_layout (pair t*K + k, or -1)
 *   route_weights  [cap] fp32 out: topk_w[row_src[r]] where row_src[r] >= 0,
 *                  else 0 (padding rows and unused capacity)
 * A row_src entry >= S*K is skipped (written 0) and sets MOE_STATUS_BAD_SLOT.
 * Host checks: S >= 0, 1 <= K <= MOE_MAX_TOPK, 0 <= cap < 2^31, 4-byte aligned
 * pointers.  One kernel; no synchronisation; status may be NULL.
 */
MOE_API int moe_dispatch_route_weights(const float *topk_w, const int32_t *row_src, int S, int K, int64_t cap,
                                       float *route_weights, int32_t *status, void *stream);

/*
 * Router variant: sigmoid scores, a selection-only bias and group-limited
 * top-K -- the router of the DeepSeek-V3 report, which "Efficient and portable
 * mixture-of-experts communication" cites; the pages give no detail, so this
 * is the plainest reading:
 *   s_e = sigmoid(l_e);  c_e = s_e + bias_e (bias [E] fp32, or NULL: c = s)
 *   n_group > 1: experts form n_group contiguous groups of E/n_group; a group's
 *     score is its largest c plus its second largest c; the topk_group best
 *     groups (ties: lower group) are kept, the others excluded
 *   topk_idx: the K largest c among kept experts (descending; ties: lower id)
 *   topk_w:  s_{e_k}, divided by sum_k s_{e_k} (k order) when normalize != 0,
 *            then multiplied by scale
 * All fp32; exp comes from IEEE basic operations (Cody-Waite reduction and a
 * degree-7 polynomial, within 2 ulp of exp), so results are reproducible.
 * Host checks: those of moe_route_topk, plus 1 <= n_group <= MOE_MAX_GROUPS,
 * E % n_group == 0, and for n_group > 1: E/n_group >= 2,
 * 1 <= topk_group <= n_group, topk_group * E / n_group >= K.
 */
#define MOE_MAX_GROUPS 32
MOE_API int moe_route_sigmoid_grouped(const float *logits, const float *bias, int S, int E, int K, int n_group,
                                      int topk_group, int normalize, float scale, int32_t *topk_idx,
                                      float *topk_w, void *stream);

/*
 * Bytes of scratch memory moe_dispatch_layout needs for these sizes
 * (a host-side query; no device work).  Returns 0 for invalid sizes.
 */
MOE_API size_t moe_dispatch_layout_workspace(int S, int E, int K);

/*
 * Per-expert histogram and prefix scan into the dispatched layout.
 * [moonep] core API: dispatch yields tokens_per_expert and cu_seqlens; tuning
 * parameters: expert groups padded to token_padding rows.  [pplx] Portable
 * Kernels: a fixed upper bound per (source rank, local expert) receive region
 * gives every writer a unique address without synchronisation; experts are
 * split over ranks in blocks of E/R.  [pplx] Dispatch: the receiver records,
 * per routed token, where it came from, for the combine.
 *
 * With pairs i = t*K + k taken in ascending order:
 *   counts[e]       [E]   int32  number of pairs routed to expert e (tokens_per_expert)
 *   offsets[e]      [E+1] int32  exclusive scan of the padded counts
 *                                pc[e] = P ? ceil(counts[e]/P)*P : counts[e] (cu_seqlens)
 *   rank_offsets[r] [R+1] int32  offsets[r*E/R]: first row of logical rank r
 *   slot_of[t,k]    [S,K] int32  offsets[e] + number of earlier pairs with the same
 *                                expert (stable: ascending token, then k); -1 if the
 *                                pair was dropped (bad index or overflow)
 *   row_src[s]      [cap] int32  the pair i with slot_of[i] == s, else -1 (padding rows
 *                                and rows past offsets[E])
 * The order inside an expert segment is one the pages leave free; ascending
 * pair order makes the layout deterministic.
 *
 * workspace: device scratch of at least moe_dispatch_layout_workspace(S,E,K)
 *   bytes, 256-byte aligned, owned by the caller.  Its first 256 bytes (the
 *   grid-synchronisation header) must be zero before the first call; every
 *   call that completes leaves them ready for the next one, so one zero-filled
 *   workspace serves any number of calls on one stream, whatever their sizes.
 *   Do not modify it between calls.  After a call that reported
 *   MOE_STATUS_TIMEOUT, zero the header again.  Calls that may run
 *   concurrently need separate workspaces.
 * Device status: MOE_STATUS_BAD_INDEX (pair dropped, not counted),
 *   MOE_STATUS_OVERFLOW (offsets[E] > cap; pairs whose slot would be >= cap
 *   get slot_of = -1).
 * Host checks: S >= 0, 1 <= E <= MOE_MAX_EXPERTS, 1 <= K <= MOE_MAX_TOPK, R >= 1,
 *   E % R == 0, token_padding >= 0, 0 <= cap < 2^31, S*K < 2^31, workspace large
 *   enough and aligned, non-NULL outputs.
 */
MOE_API int moe_dispatch_layout(const int32_t *topk_idx, int S, int E, int K, int R, int token_padding,
                        int32_t *counts, int32_t *offsets, int32_t *rank_offsets, int32_t *slot_of,
                        int32_t *row_src, int64_t cap, void *workspace, size_t workspace_bytes,
                        int32_t *status, void *stream);

/*
 * Dispatch: scatter each token row into the rows its pairs were given.
 * [pplx] Dispatch: tokens (with block scaling factors when quantised) are
 * packed and laid out contiguously per expert for the grouped GEMM.
 * [deepep] Technical overview: the dispatch may carry FP8.
 *
 *   x        [S, H]   dtype (MOE_DTYPE_F32 / MOE_DTYPE_BF16), read
 *   slot_of  [S, K]   int32, read; negative entries are skipped
 *   quant == MOE_QUANT_NONE:
 *     xd     [cap, H] dtype: xd[slot_of[t,k], :] = x[t, :] (bit copy); xs must be NULL
 *   quant == MOE_QUANT_FP8_E4M3_B128 (H % 128 == 0):
 *     xd     [cap, H] uint8 e4m3 codes, xs [cap, H/128] fp32 scales.  For block j
 *            (channels 128j..128j+127) of row t: amax = max |x| (fp32),
 *            s = amax / 448 (IEEE fp32 division), q = e4m3(x / s) with x / s an
 *            IEEE fp32 division rounded to nearest even and saturated to +-448;
 *            s == 0 gives signed zeros.  Every copy of a token carries the same
 *            bytes and scales.
 * Rows no pair maps to (padding) are not written.
 * Device status: MOE_STATUS_BAD_SLOT for a slot >= cap (skipped).
 * Host checks: S >= 0, H >= 1, 1 <= K <= MOE_MAX_TOPK, dtype/quant known, row
 * and alignment rules above, xs NULL iff quant == MOE_QUANT_NONE.
 */
MOE_API int moe_dispatch(const void *x, int dtype, int S, int H, int K, const int32_t *slot_of, int quant,
                 void *xd, float *xs, int64_t cap, int32_t *status, void *stream);

/*
 * Combine: gather each token's K expert output rows, weight them by the router
 * weights, and fuse the FarSkip-Collective dual-residual epilogue.
 * [pplx] Combine: the receiver reads the payloads the routing table names and
 * takes their router-weighted sum.  [farskip] the dual residual stream:
 *   residual_no_routed = residual + shared_out
 *   residual           = residual + mlp_output,  mlp_output = shared_out + routed
 *
 *   y          [cap, H] dtype, read (expert outputs in dispatched order)
 *   slot_of    [S, K] int32, topk_w [S, K] fp32, read
 *   shared_out [S, H] dtype or NULL;  residual [S, H] dtype or NULL
 *   residual_out           [S, H] dtype, written
 *   residual_no_routed_out [S, H] dtype or NULL, written; allowed only when both
 *                          shared_out and residual are given
 * Per element, in fp32, in this order:
 *   acc = 0; for k = 0..K-1 with 0 <= slot < cap: acc = fma(w[t,k], y[slot,h], acc)
 *   m = shared + acc (or acc);  out = residual + m (or m);  rnr = residual + shared
 * and each output rounded once to dtype (bf16: nearest even).
 * residual_out may equal residual (in place); no other buffers may overlap.
 * Device status: MOE_STATUS_BAD_SLOT for a slot >= cap (skipped).
 * Host checks: S >= 0, H >= 1, 1 <= K <= MOE_MAX_TOPK, dtype known, row and
 * alignment rules, residual_no_routed_out only with both shared_out and residual.
 */
MOE_API int moe_combine_dual_residual(const void *y, int dtype, int S, int H, int K, int64_t cap,
                              const int32_t *slot_of, const float *topk_w, const void *shared_out,
                              const void *residual, void *residual_out,
                              void *residual_no_routed_out, int32_t *status, void *stream);

/*
 * Combine over FP8 expert outputs: moe_combine_dual_residual with y given as
 * e4m3 codes plus one fp32 scale per 128-channel block -- the format of the FP8
 * dispatch ("Efficient and portable mixture-of-experts communication",
 * Dispatch: tokens travel with their block scaling factors).  Each gathered
 * element is dequantised as y = e4m3_value(q) * scale (an fp32 product); the
 * accumulation (fp32, ascending k) and the epilogue are those of
 * moe_combine_dual_residual, whose shared_out / residual / outputs here have
 * type `dtype`.
 *   yq [cap, H] uint8 e4m3 (16-byte aligned), ys [cap, H/128] fp32 (16-byte aligned)
 * Host checks as for moe_combine_dual_residual, plus H % 512 == 0.
 */
MOE_API int moe_combine_fp8_dual_residual(const uint8_t *yq, const float *ys, int dtype, int S, int H, int K,
                                          int64_t cap, const int32_t *slot_of, const float *topk_w,
                                          const void *shared_out, const void *residual, void *residual_out,
                                          void *residual_no_routed_out, int32_t *status, void *stream);

/* ------------------------------------------------------------------------ */
/* Backward of the path (training).  "MoonEP developer guide", core API      */
/* example: the backward pass reuses the forward plan -- the gradient of the  */
/* combine is dispatched through it and the gradient of the dispatch is       */
/* combined back.  The same layout (slot_of) and weights are passed in.       */
/* ------------------------------------------------------------------------ */

/*
 * Backward of moe_combine_dual_residual.  With g = dL/d(residual_out) and
 * gn = dL/d(residual_no_routed_out) (NULL: zero), per token t and pair k with
 * 0 <= slot < cap:
 *   grad_y    [cap, H] dtype  grad_y[slot] = w[t,k] * g[t]   (fp32 product, rounded
 *                             once; rows no pair maps to are not written)
 *   grad_w    [S, K] fp32     <y[slot], g[t]>  (fp32 accumulation in a fixed order;
 *                             0 for skipped pairs)
 *   grad_skip [S, H] dtype or NULL  g + gn: the gradient of both `residual` and
 *                             `shared_out` (the forward adds each once to each stream)
 * Layout, alignment and host checks as for the forward call; y is read.
 * Device status: MOE_STATUS_BAD_SLOT for a slot >= cap (skipped), MOE_STATUS_TIMEOUT.
 */
MOE_API int moe_combine_dual_residual_backward(const void *grad_out, const void *grad_no_routed,
                                               const void *y, int dtype, int S, int H, int K,
                                               int64_t cap, const int32_t *slot_of,
                                               const float *topk_w, void *grad_y, float *grad_w,
                                               void *grad_skip, int32_t *status, void *stream);

/*
 * Backward of moe_dispatch: every copy of token t carried x[t], so
 *   grad_x[t] = sum over k with 0 <= slot < cap of grad_xd[slot]   (fp32, ascending k,
 *               rounded once; zero when no copy is valid)
 * For the FP8 dispatch the quantiser is passed straight through: grad_xd holds
 * the gradients of the dequantised rows, in the activation dtype.
 *   grad_xd [cap, H] dtype (read), grad_x [S, H] dtype (written).
 */
MOE_API int moe_dispatch_backward(const void *grad_xd, int dtype, int S, int H, int K, int64_t cap,
                                  const int32_t *slot_of, void *grad_x, int32_t *status, void *stream);

/*
 * Backward of moe_route_topk through the gating softmax:
 *   grad_logits [S, E] fp32 (written, dense): w_k * (gw_k - sum_j w_j gw_j) at the
 *   selected expert e_k, 0 elsewhere (the selection is piecewise constant).
 * topk_idx, topk_w as produced by moe_route_topk; grad_w [S, K] fp32 = dL/dw.
 * Ids outside [0, E) are skipped.  Host checks as for moe_route_topk.
 */
MOE_API int moe_route_topk_backward(const int32_t *topk_idx, const float *topk_w, const float *grad_w,
                                    int S, int E, int K, float *grad_logits, void *stream);

/*
 * moe_dispatch_layout_static: the same layout as moe_dispatch_layout, for a
 * caller that cannot allocate device memory where it makes this call -- e.g. a
 * host framework or engine plugin that owns all device memory up front and
 * forbids allocation while it executes, or a latency-critical loop that must
 * not pay for cudaMalloc, which may synchronise the device.  (The pages have
 * no counterpart; this is a convenience of this library.)
 *
 * Arguments, outputs, device status and host checks are those of
 * moe_dispatch_layout without `workspace` / `workspace_bytes`.  The scratch is
 * a MOE_STATIC_LAYOUT_SCRATCH_BYTES array inside the library, held by every
 * GPU that loads the library until the process exits; sizes with
 * moe_dispatch_layout_workspace(S, E, K) > MOE_STATIC_LAYOUT_SCRATCH_BYTES
 * are refused with MOE_ERR_SCRATCH_TOO_SMALL (the limit is about 2 million
 * (token, k) pairs at E = 256, 8 million at E = 64).  Nothing is allocated: no
 * cudaMalloc, no cudaFree.
 *
 * The first call on a device looks up the array's device address there
 * (cudaGetSymbolAddress, with that device current), so make that first call
 * before any stream capture.  Every call on a device shares the one array and
 * clears its zero-initialised part on `stream` first; calls whose work may
 * overlap on the GPU (other streams, other host threads) race on it and must
 * be serialised by the caller.
 */
#define MOE_STATIC_LAYOUT_SCRATCH_BYTES (1 << 20)
MOE_API int moe_dispatch_layout_static(const int32_t *topk_idx, int S, int E, int K, int R,
                                       int token_padding, int32_t *counts, int32_t *offsets,
                                       int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src,
                                       int64_t cap, int32_t *status, void *stream);

/*
 * moe_route_dispatch: moe_route_topk, moe_dispatch_layout and moe_dispatch in
 * one call -- router top-K gating ([pplx] Introduction), the padded
 * expert-contiguous layout ([pplx] Portable Kernels, Dispatch; [moonep] core
 * API example, tuning parameters) and the row scatter, optionally FP8
 * ([pplx] Dispatch; [deepep] Technical overview).  Every output is exactly
 * what the three calls would write (same router, same stable counting sort,
 * same FP8 arithmetic):
 *   topk_idx, topk_w   as moe_route_topk
 *   counts, offsets, rank_offsets, slot_of, row_src   as moe_dispatch_layout
 *                      on those ids (R, token_padding, cap)
 *   xd, xs             as moe_dispatch of x (dtype, quant) with that slot_of
 * The token rows x do not depend on the routing, so when the batch's share of
 * each SM fits in shared memory (for example S <= 4144 tokens of H = 7168 bf16
 * with FP8 on a 148-SM B200) the call is ONE cooperative kernel that reads and
 * quantises x while it routes, keeps the rows in shared memory until their
 * slots are known and then stores them; otherwise it launches the three
 * separate kernels.  moe_route_dispatch_kernels tells which.
 *
 * workspace: device scratch of at least moe_route_dispatch_workspace(S, E, K)
 *   bytes, 256-byte aligned, owned by the caller.  ALL of it must be zero
 *   before the first call (the fused kernel keeps per-CTA arrival marks there,
 *   past the part moe_dispatch_layout uses); every completed call leaves it
 *   ready for the next one, whatever the sizes; after a MOE_STATUS_TIMEOUT
 *   zero all of it again.  Do not modify it between calls; concurrent calls
 *   need separate workspaces.  The same buffer also serves
 *   moe_dispatch_layout (for the same or smaller S, E, K).
 * Device status: the union of the three calls' bits, and MOE_STATUS_TIMEOUT
 *   if a bounded wait of the fused kernel ran out.
 * Host checks: the union of the three calls' checks.
 */
MOE_API size_t moe_route_dispatch_workspace(int S, int E, int K);
MOE_API int moe_route_dispatch(const float *logits, const void *x, int dtype, int S, int H, int E, int K, int R,
                               int token_padding, int quant, int32_t *topk_idx, float *topk_w, int32_t *counts,
                               int32_t *offsets, int32_t *rank_offsets, int32_t *slot_of, int32_t *row_src,
                               void *xd, float *xs, int64_t cap, void *workspace, size_t workspace_bytes,
                               int32_t *status, void *stream);

/*
 * Kernels moe_route_dispatch launches for these sizes on the current device:
 * 1 (the fused kernel) or 3 / 4 (router, layout in 1 or 2 kernels, dispatch).
 * No launch happens.  Returns -1 on a CUDA error, 0 for invalid sizes.
 */
MOE_API int moe_route_dispatch_kernels(int S, int H, int E, int K, int dtype, int quant);

/* ------------------------------------------------------------------------ */
/* Expert parallelism over W ranks (one GPU each).  Each rank routes its own  */
/* tokens and builds its local layout with R = W (moe_route_topk,             */
/* moe_dispatch_layout, P = 0): that layout is its send buffer, rank-major.   */
/* The ranks exchange their per-expert counts (an all-gather of [E] int32),   */
/* and each derives the same receive plan with moe_ep_plan; rows then move    */
/* between ranks (NCCL point-to-point, one segment per (peer, expert)) and    */
/* the combine runs on each source rank over its own send-order buffer.       */
/* ------------------------------------------------------------------------ */

/*
 * Receive plan of expert parallelism (host memory, host computation, no GPU).
 * [pplx] Portable Kernels: experts in blocks of E/W per rank, a fixed region
 * per (source rank, local expert) in the receiver's buffer; [pplx] Dispatch:
 * the rows of one expert contiguous at the receiver; [moonep] core API
 * example: Buffer(S, H, K, E, num_ep_ranks), token_padding.
 *
 *   counts         [W, E] int32 (host, read): counts[s][e] = pairs of source
 *                  rank s routed to expert e (its layout's `counts`)
 *   expert_offsets [E + 1] int32 (host, written): the padded offsets of the
 *                  whole batch, rank-major -- exactly moe_dispatch_layout's
 *                  `offsets` for all ranks' tokens taken in rank order
 *   recv_offsets   [W, W, E/W] int32 (host, written): recv_offsets[d][s][j] is
 *                  the first row, in rank d's receive buffer, of source rank
 *                  s's rows of expert d*E/W + j (they follow in source order)
 *   recv_rows      [W] int32 (host, written): rows of rank d's receive buffer
 *                  (padding included)
 * Returns MOE_OK, or MOE_ERR_INVALID_ARG for W < 1, E outside
 * [1, MOE_MAX_EXPERTS], E % W != 0, token_padding < 0, a negative count, a
 * total past 2^31 - 1 rows, or a NULL pointer.
 */
MOE_API int moe_ep_plan(const int32_t *counts, int W, int E, int token_padding, int32_t *expert_offsets,
                        int32_t *recv_offsets, int32_t *recv_rows);

/* Human-readable name of a return code (static string, host). */
MOE_API const char *moe_error_string(int code);

/* Row capacity that always fits the padded layout: S*K + E*max(P-1, 0) (host). */
MOE_API int64_t moe_capacity(int S, int E, int K, int token_padding);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTE_H */
