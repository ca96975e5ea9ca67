/*
 * moe.h -- C ABI of libmoe: the single-GPU core of an expert-parallel
 * mixture-of-experts layer on NVIDIA B200 (sm_100a).
 *
 * One MoE layer, as "Expert parallelism and all-to-all" walks through it
 * (section "Walking through one MoE layer"): the router gives every token
 * k (expert, weight) picks; dispatch sends each token's hidden vector to
 * the owners of its experts; each owner runs its local experts on what it
 * received as one grouped matrix multiply; combine returns the outputs to
 * the token's home row as a router-weighted sum.  On one GPU, the logical
 * expert-parallel ranks ("Expert parallelism" (Transformers docs), section
 * "How the sizes combine": rank r of W owns experts [r*E/W, (r+1)*E/W))
 * only fix the slab layout of the permuted buffer; no collective is issued.
 *
 *   moe_route_topk       logits[T,E]                 -> topk_idx[T,k], topk_w[T,k]
 *   moe_dispatch_layout  topk_idx[T,k]               -> counts, offsets, rank slabs,
 *                                                       slot_of_pair[N], pair_of_slot[N]
 *   moe_permute          x[T,H], slot_of_pair        -> xp[N,H] (+ FP8 block scales)
 *   moe_grouped_gemm     xp, offsets, W13, W2        -> h[N,I], y[N,H]  (SwiGLU FFN)
 *   moe_combine          y, slot_of_pair, topk_w     -> out[T,H]
 *   moe_layer_forward    the five calls in one, with per-step events
 *
 * with N = T*k routed pairs; pair p = t*k + j is token t's j-th pick.
 * Variants the pages discuss: moe_route_topk_grouped (at most M expert
 * groups per token), moe_dispatch_layout_capacity (fixed slabs of C rows per
 * expert, dropping the rest), an FP8 combine payload (y as e4m3 + block
 * scales), and moe_dispatch_layout_noalloc (the layout without a caller
 * workspace).
 *
 * Conventions shared by every call:
 *  - All arrays are dense, row-major, and live in device memory (except
 *    where a call says otherwise).  Index arrays are int32.
 *  - The caller allocates and owns every buffer, including workspaces and
 *    the device status word.  The library allocates nothing, frees
 *    nothing and never synchronises, except moe_check_status and the
 *    diagnostic moe_diag_gemm_clock.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call only enqueues work on it and returns; the chain of calls has no
 *    host synchronisation, so it can be captured in a CUDA graph.
 *  - Arguments are validated on the host before anything is enqueued.  An
 *    invalid call returns MOE_ERR_INVALID_ARG (or MOE_ERR_UNSUPPORTED for a
 *    valid request beyond the kernels' limits) and touches no output.  This
 *    follows the pages' own rule of refusing a bad configuration up front
 *    rather than silently falling back ("Expert parallelism" (Transformers
 *    docs), "Overriding the plans"; the expert-parallel-plan ValueError of
 *    transformers' distributed mixin).
 *  - T == 0 is a valid, empty batch ("token slices may be uneven or
 *    empty", Transformers docs, "With tensor parallelism"); experts that
 *    receive no rows are valid too.
 *  - Errors found on the device (an expert id outside [0, E); a bounded
 *    wait that ran out) are OR-ed into the caller's int32 status word
 *    `dev_status` and the call still returns MOE_OK; moe_check_status
 *    reports them.  A failed kernel launch returns MOE_ERR_CUDA.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad dtype combination */
    MOE_ERR_UNSUPPORTED = 2, /* valid but beyond the kernels' limits (E > 1024, k > 16) */
    MOE_ERR_BAD_INDEX = 3,   /* device: an expert id outside [0, E) was skipped */
    MOE_ERR_TIMEOUT = 4,     /* device: a bounded wait ran out; results invalid */
    MOE_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
    MOE_ERR_OVERFLOW = 6     /* device: a row fell outside a receive buffer and was skipped */
} moe_status;

typedef enum moe_dtype {
    MOE_F32 = 0,  /* IEEE binary32 */
    MOE_BF16 = 1, /* bfloat16 */
    MOE_E4M3 = 2  /* OCP FP8 E4M3 (no infinities, max 448): payloads (xp, y) only */
} moe_dtype;

/* Bits of the device status word. */
#define MOE_DEV_BAD_INDEX 0x1
#define MOE_DEV_TIMEOUT 0x2
#define MOE_DEV_OVERFLOW 0x4

/* Kernel limits (MOE_ERR_UNSUPPORTED beyond them). */
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 16

/*
 * moe_route_topk -- router top-k with softmax weights.
 * Source: "Expert parallelism and all-to-all", "Walking through one MoE
 * layer", step 1 (every token gets a list of (expert, weight) picks); the
 * Transformers docs' (top_k_index, top_k_weights) pair ("Adding an
 * implementation").
 *
 *   logits   [T, E] fp32, device, read only.
 *   topk_idx [T, k] int32, device, written: token t's picks in order of
 *            (logit descending, expert id ascending); ties go to the
 *            lower expert id, -0 and +0 compare equal.
 *   topk_w   [T, k] fp32, device, written: softmax over the k picked
 *            logits (equal to the full softmax over E, restricted to the
 *            picks and renormalised).
 * Requires 1 <= k <= E, E <= MOE_MAX_EXPERTS, k <= MOE_MAX_TOPK.  Logits
 * must be finite (NaN ordering is not defined).
 */
moe_status moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k,
                          int32_t* topk_idx, float* topk_w, void* stream);

/*
 * moe_route_topk_grouped -- moe_route_topk restricted to at most
 * `max_groups` expert groups per token.
 *
 * Source: "Expert Parallelism" (aiwiki), "Hiding the latency",
 * topology-aware routing: DeepSeek-V3's router sends each token to at most
 * 4 nodes, bounding the inter-node fan-out.  The page does not say how the
 * nodes are chosen; this library reads it as: the E experts form `groups`
 * equal groups of consecutive ids (a node holds a logical rank's block); a
 * group's score is its largest logit; each token keeps the `max_groups`
 * groups with the highest scores (ties: lower group id) and takes its top k
 * among their experts with the rule of moe_route_topk (logit descending,
 * expert id ascending); the weights are the softmax over the k picks.
 * max_groups == groups gives moe_route_topk's result.
 *
 * Arguments as moe_route_topk.  Requires groups | E, 1 <= max_groups <=
 * groups, k <= max_groups * E / groups (MOE_ERR_INVALID_ARG otherwise) and
 * groups <= 32 (MOE_ERR_UNSUPPORTED).
 */
moe_status moe_route_topk_grouped(const float* logits, int64_t T, int32_t E, int32_t k,
                                  int32_t groups, int32_t max_groups, int32_t* topk_idx,
                                  float* topk_w, void* stream);

/*
 * moe_dispatch_layout -- the dispatch plan: a per-expert histogram, its
 * exclusive scan, and a stable expert-major permutation of the pairs.
 * Source: "Expert Parallelism" (aiwiki), "Implementation": sort the tokens
 * by destination so each peer's rows are one contiguous slab, and count
 * them per rank (bincount of idx // per_rank); the sort is taken as stable
 * (ties by pair index).  Ownership: rank r owns experts [r*E/W, (r+1)*E/W)
 * (Transformers docs, "How the sizes combine"), so the expert-major order
 * is also rank-major and rank r's slab is [rank_offsets[r],
 * rank_offsets[r+1]) -- exactly the send buffer of a dispatch all-to-all.
 *
 *   topk_idx       [T, k] int32, device, read only.
 *   expert_counts  [E] int32, written: rows routed to each expert.
 *   expert_offsets [E+1] int32, written: exclusive scan of the counts.
 *   rank_offsets   [W+1] int32, written: expert_offsets[r*E/W].
 *   slot_of_pair   [T*k] int32, written: the slot (row of the permuted
 *                  buffer) of pair p; -1 for a pair with a bad expert id.
 *   pair_of_slot   [T*k] int32, written: inverse map; slots past
 *                  expert_offsets[E] hold -1.
 *   workspace      device scratch of at least
 *                  moe_dispatch_layout_workspace_bytes(T, k, E) bytes, 16-byte
 *                  aligned; no initial contents needed; clobbered.
 *   dev_status     int32 device word; MOE_DEV_BAD_INDEX is OR-ed in when a
 *                  pair's expert id is outside [0, E) (the pair is skipped),
 *                  MOE_DEV_TIMEOUT if the scan's bounded wait ran out.
 * Requires 1 <= k, 1 <= W <= E, E % W == 0 (ep_size must divide the number
 * of experts, Transformers docs, "Adding an implementation"), E <=
 * MOE_MAX_EXPERTS, T*k < 2^31.
 */
size_t moe_dispatch_layout_workspace_bytes(int64_t T, int32_t k, int32_t E);
moe_status moe_dispatch_layout(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                               int32_t W, int32_t* expert_counts, int32_t* expert_offsets,
                               int32_t* rank_offsets, int32_t* slot_of_pair,
                               int32_t* pair_of_slot, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_dispatch_layout_capacity -- the dispatch layout with a fixed capacity
 * of C rows per expert; the pairs that do not fit are dropped.
 *
 * Source: "Expert Parallelism" (aiwiki), "Implementation", closing note:
 * with fixed buffers every destination's size is known in advance (no
 * count exchange before the payload), and the tokens that do not fit are
 * the price.  The page gives neither the size nor the drop rule; this
 * library reads it as: expert e owns the fixed slab [e*C, (e+1)*C) of the
 * permuted buffer; its pairs, in pair order (the stable order of
 * moe_dispatch_layout), fill the slab from the top, and the pairs past the
 * C-th are dropped.  A dropped pair contributes nothing to the combine.
 *
 *   capacity       C >= 0 rows per expert (e.g. ceil(factor * T*k / E)).
 *   expert_counts  [E] int32, written: rows kept per expert, min(count, C).
 *   expert_offsets [E+1] int32, written: e*C (fixed).
 *   rank_offsets   [W+1] int32, written: (r*E/W)*C (fixed).
 *   slot_of_pair   [T*k] int32, written: e*C + the pair's rank among
 *                  expert e's pairs; -1 for a dropped pair or a bad id.
 *   pair_of_slot   [E*C] int32, written: inverse map; slab rows past an
 *                  expert's kept pairs hold -1.
 *   n_dropped      int32 device word or NULL: written with the number of
 *                  dropped pairs (bad ids not included).
 *   workspace, workspace_bytes, dev_status, stream: as moe_dispatch_layout.
 * Requirements as moe_dispatch_layout, plus E*C < 2^31.  C < 0 returns
 * MOE_ERR_INVALID_ARG.  The segments handed to moe_grouped_gemm are then
 * expert_offsets with expert_counts (the rows each expert computes).
 */
moe_status moe_dispatch_layout_capacity(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                                        int32_t W, int32_t capacity, int32_t* expert_counts,
                                        int32_t* expert_offsets, int32_t* rank_offsets,
                                        int32_t* slot_of_pair, int32_t* pair_of_slot,
                                        int32_t* n_dropped, void* workspace,
                                        size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_dispatch_layout_noalloc -- moe_dispatch_layout for callers that cannot
 * allocate device memory.  The pages have no counterpart: this is a
 * convenience of this library, not a step of the method.
 *
 * Some callers cannot hand the library a workspace: cudaMalloc may
 * synchronise the device and is not allowed while a stream is being
 * captured, and some host frameworks keep all device memory in their own
 * allocator and give extensions no way to ask for scratch.  This variant
 * takes the same inputs and outputs as moe_dispatch_layout, minus the
 * workspace, and computes exactly the same results.
 *
 *   - Its scratch is one fixed array inside the library, of
 *     moe_dispatch_layout_noalloc_max_scratch_bytes() bytes (2 MiB), which
 *     every GPU that loads the library holds until the process exits.
 *   - Sizes whose scratch would not fit (E * ceil(T*k / 2048) above about
 *     262,000, e.g. more than ~2 million pairs at E = 256) return
 *     MOE_ERR_UNSUPPORTED; moe_dispatch_layout handles those.
 *   - It allocates nothing.  The first call on each device looks up the
 *     array's device address (cudaGetSymbolAddress, with that device
 *     current), and looks it up again whenever the context current on the
 *     device is not the one of the last lookup (after cudaDeviceReset, or
 *     with another context made current); make the first call in each
 *     context before any stream capture.  A CUDA error in the lookup or the
 *     launch returns MOE_ERR_CUDA (and is printed, as for every entry point).
 *   - Every call shares the one array, so calls that overlap on the GPU
 *     (on different streams, or from different threads) race: serialise
 *     them, e.g. on one stream.  Nothing needs clearing between calls.
 *   - Its argument rules are moe_dispatch_layout's (without the workspace).
 */
size_t moe_dispatch_layout_noalloc_max_scratch_bytes(void);
moe_status moe_dispatch_layout_noalloc(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                                       int32_t W, int32_t* expert_counts,
                                       int32_t* expert_offsets, int32_t* rank_offsets,
                                       int32_t* slot_of_pair, int32_t* pair_of_slot,
                                       int32_t* dev_status, void* stream);

/*
 * moe_permute -- write every token's hidden vector into the slots of its
 * k pairs: xp[slot_of_pair[t*k + j]] = x[t] (the "sent = x[order]" of the
 * aiwiki sketch, done as a scatter so each x row is read once).
 * Source: aiwiki, "Implementation"; FP8 payload: "Expert parallelism and
 * all-to-all", "Traffic math" (FP8 activations, 1 byte per element).
 *
 *   x         [T, H] in x_dtype (MOE_F32 or MOE_BF16), device, read only.
 *   slot_of_pair [T*k] int32 from moe_dispatch_layout; pairs holding -1
 *             are skipped.
 *   xp        [T*k, H] in xp_dtype, device, written at the pairs' slots.
 *             xp_dtype == x_dtype: a bitwise copy.
 *             xp_dtype == MOE_E4M3: for each 128-element block of a token
 *             row, scale = amax/448 (fp32 IEEE division; 1 if amax == 0)
 *             and q = e4m3(x/scale) (fp32 IEEE division, round to nearest
 *             even, saturating to +-448).  Requires H % 128 == 0.
 *   xp_scales [T*k, H/128] fp32, written for MOE_E4M3 (16-byte aligned: a
 *             slot's scales are stored as 16-byte vectors), else ignored
 *             (may be NULL).
 * Requires H % 8 == 0, H > 0, k >= 1; x and xp 16-byte aligned.
 */
moe_status moe_permute(const void* x, moe_dtype x_dtype, int64_t T, int32_t H, int32_t k,
                       const int32_t* slot_of_pair, void* xp, moe_dtype xp_dtype,
                       float* xp_scales, void* stream);

/*
 * moe_grouped_gemm -- every local expert's SwiGLU FFN over its rows, as
 * one grouped GEMM ("Expert parallelism and all-to-all", "Walking through
 * one MoE layer", step 3; the Transformers docs' experts_forward; expert
 * weights stacked along the expert dimension, "GroupedGemmParallel").
 *
 * For local expert j (global expert e = expert_begin + j) and every slot s
 * in [expert_offsets[e], expert_offsets[e] + rows_e), rows_e =
 * expert_offsets[e+1] - expert_offsets[e] (or min(that, expert_counts[e])
 * when expert_counts is given: the fixed slabs of
 * moe_dispatch_layout_capacity, whose tail rows hold no pair):
 *     g = A_s W13[j, 0:I, :]^T,  u = A_s W13[j, I:2I, :]^T,
 *     h_s = silu(g) * u  (silu(g) = g / (1 + exp(-g))),
 *     y_s = h_s W2[j]^T,
 * accumulated in fp32.  A_s is the xp row; for an FP8 payload it is
 * bf16(decode(q) * scale) (fp32 product, rounded to bf16).
 *
 *   xp             [n_rows, H] in xp_dtype, device.
 *   xp_scales      [n_rows, H/128] fp32 when xp_dtype == MOE_E4M3, else NULL.
 *   expert_offsets [>= expert_begin + n_experts + 1] int32, DEVICE memory:
 *                  read by the kernels, never by the host.
 *   expert_counts  NULL, or [>= expert_begin + n_experts] int32 in DEVICE
 *                  memory: rows computed per expert (see above).
 *   w13            [n_experts, 2I, H] in w_dtype (gate rows, then up rows).
 *   w2             [n_experts, H, I] in w_dtype.
 *   h              [n_rows, I] in w_dtype, written for the experts' rows (the
 *                  down projection's operand, so it has the GEMM's dtype).
 *   y              [n_rows, H] in y_dtype, written for the experts' rows:
 *                  MOE_F32 (either path), MOE_BF16 or MOE_E4M3 (bf16 path
 *                  only).  fp32 keeps the combine within 2e-2 of a row's RMS
 *                  of the exact layer output; a bf16 y adds a second bf16
 *                  rounding before the weighted sum, which alone can take the
 *                  largest elements of a row past that bound.  MOE_E4M3 is
 *                  the FP8 combine payload ("Expert parallelism and
 *                  all-to-all", "Traffic math": 1-byte activations both
 *                  ways): per 128 outputs of a row, scale = amax/448 of the
 *                  fp32 values and the codes e4m3(y/scale), by the same rule
 *                  as moe_permute's FP8 payload; requires H % 128 == 0.
 *   y_scales       [n_rows, H/128] fp32, written when y_dtype == MOE_E4M3,
 *                  else ignored (may be NULL).
 *   workspace      device scratch of moe_grouped_gemm_workspace_bytes(...)
 *                  bytes (may be 0 / NULL when that is 0), 128-byte aligned.
 *   dev_status     int32 device word (MOE_DEV_TIMEOUT on a bounded wait
 *                  running out).
 * Dtypes: w_dtype MOE_F32 with xp MOE_F32 (CUDA-core fp32 path), or w_dtype
 * MOE_BF16 with xp MOE_BF16 or MOE_E4M3 (tensor-core path).  Requires H % 8
 * == 0, I % 8 == 0 (H % 128 == 0 for E4M3), and the offsets to be
 * non-decreasing with expert_offsets[expert_begin + n_experts] <= n_rows.
 * xp, h, y, w13, w2 must be 16-byte aligned.
 */
size_t moe_grouped_gemm_workspace_bytes(int64_t n_rows, int32_t H, int32_t I,
                                        moe_dtype xp_dtype, moe_dtype w_dtype);
moe_status moe_grouped_gemm(const void* xp, moe_dtype xp_dtype, const float* xp_scales,
                            const int32_t* expert_offsets, const int32_t* expert_counts,
                            int32_t expert_begin,
                            int32_t n_experts, int64_t n_rows, int32_t H, int32_t I,
                            const void* w13, const void* w2, moe_dtype w_dtype, void* h,
                            void* y, moe_dtype y_dtype, float* y_scales, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_pack_expert_weights -- one-time re-layout of the stacked expert
 * weights (W13 [E, 2I, H], W2 [E, H, I], bf16) into blocks of 128 rows x
 * 64 columns, each 16 KB block contiguous, in the order the grouped GEMM
 * reads them: W13 block (e, f, c) holds gate features [64f, 64f+64) and the
 * matching up features of columns [64c, 64c+64); W2 block (e, r, c) rows
 * [128r, 128r+128) of columns [64c, 64c+64).  Rows and columns past the
 * matrices are zero.  In the stacked layout a 128-row tile of one k-step is
 * 128 pieces of 128 bytes, H*2 (or I*2) bytes apart; packed, it is one
 * contiguous read.  The values are unchanged: moe_grouped_gemm_packed on the
 * packed weights computes exactly moe_grouped_gemm's results.
 *   w13, w2             stacked weights (either may be NULL to pack only
 *                       the other), 16-byte aligned, device.
 *   packed13, packed2   outputs of moe_packed_weights_bytes(E, H, I, 0) and
 *                       (..., 1) bytes, 16-byte aligned, device.
 * Requires w_dtype MOE_BF16, H % 8 == 0, I % 8 == 0.  A shard of experts
 * [a, b) packs from the stacked shard w13[a:b], w2[a:b] with E = b - a.
 */
size_t moe_packed_weights_bytes(int32_t E, int32_t H, int32_t I, int32_t which);
moe_status moe_pack_expert_weights(const void* w13, const void* w2, int32_t E, int32_t H,
                                   int32_t I, moe_dtype w_dtype, void* packed13, void* packed2,
                                   void* stream);

/*
 * moe_grouped_gemm_packed -- moe_grouped_gemm with the expert weights in
 * moe_pack_expert_weights' layout (bf16 weights; the tensor-core kernel
 * with the weights as the MMA's M operand runs at every size).  Arguments
 * and results as moe_grouped_gemm, with packed13 / packed2 in place of
 * w13 / w2 (packed for the n_experts local experts).
 */
moe_status moe_grouped_gemm_packed(const void* xp, moe_dtype xp_dtype, const float* xp_scales,
                                   const int32_t* expert_offsets, const int32_t* expert_counts,
                                   int32_t expert_begin, int32_t n_experts, int64_t n_rows,
                                   int32_t H, int32_t I, const void* packed13,
                                   const void* packed2, moe_dtype w_dtype, void* h, void* y,
                                   moe_dtype y_dtype, float* y_scales, void* workspace,
                                   size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_combine -- un-permute plus the router-weighted sum of each token's k
 * expert outputs into its home row:
 *     out[t] = sum_{j=0..k-1} topk_w[t,j] * y[slot_of_pair[t*k+j]],
 * fp32 accumulation in j order, rounded once to out_dtype; pairs holding
 * slot -1 add nothing.
 * Source: aiwiki, "Implementation" (y[order] = back, undoing the sort);
 * "Expert parallelism and all-to-all", step 4 (the home GPU takes a
 * weighted sum into the residual stream); Transformers docs (the weighted
 * expert output for each token).
 *
 *   y            [>= max slot + 1, H] in y_dtype (MOE_F32 / MOE_BF16, or MOE_E4M3
 *                codes with one scale per 128-element block: a code adds
 *                (topk_w * scale) * decode(q), the weight-scale product in
 *                fp32 once per 16 codes, then a fused multiply-add per
 *                code), device.
 *   y_scales     [>= max slot + 1, H/128] fp32 when y_dtype == MOE_E4M3
 *                (H % 128 == 0), else ignored (may be NULL).
 *   slot_of_pair [T*k] int32, device.
 *   topk_w       [T, k] fp32, device; or NULL for unit weights (rows that
 *                already carry their router weight: out = the k-way sum).
 *   out          [T, H] in out_dtype (MOE_F32 / MOE_BF16), device, written.
 * Requires H % 8 == 0, k >= 1.
 */
moe_status moe_combine(const void* y, moe_dtype y_dtype, const float* y_scales,
                       const int32_t* slot_of_pair, const float* topk_w, int64_t T, int32_t k,
                       int32_t H, void* out, moe_dtype out_dtype, void* stream);

/*
 * moe_combine_rank -- rank `rank`'s partial in the all_reduce form of the
 * layer, where no token moves: every rank holds the whole batch, runs its
 * own experts, and the ranks' per-token outputs are summed by an
 * all-reduce (Transformers docs, "Expert parallelism", "Choosing an
 * implementation", the all_reduce row).  Rank r's experts own the slots
 * [rank_offsets[r], rank_offsets[r+1]) of the layout, so
 *     partial[t] = sum over j with slot_of_pair[t*k+j] in that range of
 *                  topk_w[t,j] * y[slot_of_pair[t*k+j]],
 * fp32 accumulation in j order, unrounded fp32 result (zeros for a token
 * with no pick on the rank).  The bounds are read on the device, so the
 * call needs no host synchronisation.
 *
 *   y, y_dtype, y_scales, slot_of_pair, topk_w, T, k, H: as moe_combine.
 *   rank_offsets [world + 1] int32, device (moe_dispatch_layout's output).
 *   rank         in [0, world).
 *   partial      [T, H] fp32, device, written (16-byte aligned).
 */
moe_status moe_combine_rank(const void* y, moe_dtype y_dtype, const float* y_scales,
                            const int32_t* slot_of_pair, const float* topk_w, int64_t T,
                            int32_t k, int32_t H, const int32_t* rank_offsets, int32_t world,
                            int32_t rank, float* partial, void* stream);

/*
 * moe_reduce_partials -- the all-reduce's sum of n_partials fp32 partials
 * [n_partials, T, H] (contiguous): out = ((p[0] + p[1]) + p[2]) + ..., in
 * fp32 in rank order, rounded once to out_dtype (MOE_F32 / MOE_BF16).
 * With n_partials = 1 it is the rounding that follows an all-reduce done
 * elsewhere (for example NCCL over W GPUs, on the fp32 partials).
 * Requires H % 8 == 0; partials and out 16-byte aligned, device.
 */
moe_status moe_reduce_partials(const float* partials, int32_t n_partials, int64_t T, int32_t H,
                               void* out, moe_dtype out_dtype, void* stream);

/*
 * Expert parallelism over W ranks (W GPUs of one NVLink domain, one process
 * each; or W ranks run on one GPU).  Each rank holds its own T tokens and
 * the weights of its E/W experts [r*E/W, (r+1)*E/W) ("Expert parallelism"
 * (Transformers docs), "How the sizes combine").  One layer, per rank:
 *   1. moe_route_topk and moe_dispatch_layout on its own tokens;
 *   2. the count exchange: every rank's expert_counts gathered into
 *      counts_all [W, E] on every rank (for example an all-gather over
 *      NCCL) -- "Expert Parallelism" (aiwiki), "Implementation": peers must
 *      know how much is coming;
 *   3. moe_ep_plan: where this rank's rows land in each owner's receive
 *      buffer, and where its own local experts start in its buffer;
 *   4. moe_ep_dispatch: every routed row stored into its owner's receive
 *      buffer (the dispatch all-to-all, "The two all-to-alls");
 *   5. once every rank's dispatch has completed (a barrier across ranks):
 *      moe_grouped_gemm on the local receive buffer, expert_offsets =
 *      recv_offsets, expert_begin = 0, n_experts = E/W, the local weights;
 *   6. once every rank's GEMM has completed: moe_ep_combine, which reads
 *      each pick's output row from its owner's y buffer (the combine
 *      all-to-all) and takes the router-weighted sum.
 * Every routed row's result is the same as on one GPU: out equals
 * moe_layer_forward's on the same tokens, bit for bit.
 *
 * Receive layout (a reading: the pages' all_to_all_single delivers one
 * chunk per source rank): an owner's buffer holds its experts one after the
 * other, and inside an expert the rows of rank 0, then rank 1, ..., each in
 * the sender's slot order, so each local expert is one contiguous segment.
 */

/*
 * moe_ep_plan -- this rank's dispatch plan from the exchanged counts.
 *   counts_all   [W, E] int32, device: rows rank s routes to expert e.
 *   send_base    [E] int32, device, written: the row of expert e's owner's
 *                receive buffer where this rank's rows for e begin.
 *   recv_offsets [E/W + 1] int32, device, written: where local expert j
 *                begins in this rank's receive buffer; recv_offsets[E/W] is
 *                the number of rows it receives.
 *   dev_status   MOE_DEV_BAD_INDEX if a count is negative (read as 0).
 * Requires W | E, 0 <= rank < W, W <= 64, E <= MOE_MAX_EXPERTS.
 */
moe_status moe_ep_plan(const int32_t* counts_all, int32_t W, int32_t E, int32_t rank,
                       int32_t* send_base, int32_t* recv_offsets, int32_t* dev_status,
                       void* stream);

/*
 * moe_ep_dispatch -- the dispatch all-to-all as stores: for each of this
 * rank's routed pairs p = t*k + j (slot s = slot_of_pair[p] >= 0, expert e =
 * topk_idx[p]), row x[t] (or its FP8 payload, by moe_permute's rule) is
 * written to row send_base[e] + (s - expert_offsets[e]) of the receive
 * buffer of rank e / (E/W).
 *   x, x_dtype, T, H, k     as moe_permute.
 *   topk_idx, slot_of_pair, expert_offsets   this rank's route and layout.
 *   send_base               from moe_ep_plan.
 *   recv_rows, recv_scales  HOST arrays of W device pointers: every rank's
 *                           receive buffer [rows_capacity, H] in
 *                           payload_dtype, and for MOE_E4M3 its block scales
 *                           [rows_capacity, H/128] fp32 (16-byte aligned; may
 *                           be NULL otherwise).  Across GPUs these are
 *                           peer-mapped pointers.
 *   rows_capacity           rows of every receive buffer; a row at or past
 *                           it is skipped and MOE_DEV_OVERFLOW flagged.
 * payload_dtype is x_dtype or MOE_E4M3.  The call only writes; the owners
 * may read their buffers once every rank's dispatch has completed.
 */
moe_status moe_ep_dispatch(const void* x, moe_dtype x_dtype, int64_t T, int32_t H, int32_t k,
                           const int32_t* topk_idx, const int32_t* slot_of_pair,
                           const int32_t* expert_offsets, const int32_t* send_base, int32_t E,
                           int32_t W, void* const* recv_rows, float* const* recv_scales,
                           moe_dtype payload_dtype, int64_t rows_capacity, int32_t* dev_status,
                           void* stream);

/*
 * moe_ep_combine -- the combine all-to-all as loads, fused with the
 * weighted sum: out[t] = sum_j topk_w[t,j] * y_owner[row(p)], with row(p)
 * as in moe_ep_dispatch and y_owner the owner's expert outputs (written by
 * its moe_grouped_gemm at its receive rows), fp32 accumulation in j order,
 * rounded once to out_dtype (moe_combine's rule).
 *   y_rows, y_scales   HOST arrays of W device pointers: every rank's y
 *                      [rows_capacity, H] in y_dtype (and its block scales
 *                      for MOE_E4M3).
 *   rows_capacity      rows of every y buffer (MOE_DEV_OVERFLOW past it).
 * Other arguments as moe_ep_dispatch and moe_combine.
 */
moe_status moe_ep_combine(void* const* y_rows, float* const* y_scales, moe_dtype y_dtype,
                          const int32_t* topk_idx, const int32_t* slot_of_pair,
                          const int32_t* expert_offsets, const int32_t* send_base,
                          const float* topk_w, int64_t T, int32_t k, int32_t H, int32_t E,
                          int32_t W, int64_t rows_capacity, void* out, moe_dtype out_dtype,
                          int32_t* dev_status, void* stream);

/*
 * Buffer sharing between processes for the expert-parallel tables: a rank
 * exports each receive / output buffer as a record of
 * moe_ipc_handle_bytes() bytes (the CUDA IPC handle of the allocation that
 * holds it, and the buffer's offset inside that allocation), sends the
 * records to the other ranks by any host means, and every rank maps the
 * others' buffers with moe_ipc_import; the mapped addresses (peer memory
 * over NVLink) go into the W-entry tables.  moe_ipc_close unmaps.  The
 * buffer must come from cudaMalloc (for example PyTorch's default caching
 * allocator, not its expandable segments); no multicast object is created.
 *   moe_ipc_export: ptr a device pointer of this process; record written
 *                   (host memory).
 *   moe_ipc_import: record from another process; *ptr receives the mapped
 *                   address of the same buffer (cudaIpcOpenMemHandle, peer
 *                   access enabled lazily).  A record of this same process
 *                   cannot be imported (CUDA refuses it).
 *   moe_ipc_close:  the record and the address moe_ipc_import gave.
 * CUDA failures return MOE_ERR_CUDA.
 */
size_t moe_ipc_handle_bytes(void);
moe_status moe_ipc_export(const void* ptr, void* record);
moe_status moe_ipc_import(const void* record, void** ptr);
moe_status moe_ipc_close(const void* record, void* ptr);

/*
 * moe_layer_forward -- the whole hot path in one call: moe_route_topk,
 * moe_dispatch_layout, moe_permute, moe_grouped_gemm (every expert, local
 * expert j = global expert j) and moe_combine, in that order on `stream`,
 * with exactly the semantics of the five calls ("Expert parallelism and
 * all-to-all", "Walking through one MoE layer", steps 1-4).  All five
 * calls' arguments are validated before the first launch.
 *
 *   logits [T, E] fp32 and x [T, H] (x_dtype) are the layer's inputs;
 *   w13 / w2 the stacked expert weights (w_dtype); out [T, H] in x_dtype.
 *   b holds every intermediate buffer and workspace (device, caller
 *   owned); b->xp is in payload_dtype (x_dtype or MOE_E4M3), b->y in
 *   y_dtype.
 *   opts (may be NULL: capacity -1, route_groups 0, fused_gather 0,
 *   all_reduce_form 0, packed_weights 0, weights_in_gemm 0):
 *     capacity: -1 for the dropless layout (moe_dispatch_layout; the
 *     permuted buffers have T*k rows), or C >= 0 for fixed slabs of C rows
 *     per expert (moe_dispatch_layout_capacity; E*C rows, dropped pairs
 *     add nothing, b->n_dropped receives their number when not NULL);
 *     route_groups, route_max_groups: 0 for plain routing (moe_route_topk),
 *     or G and M for moe_route_topk_grouped.
 *     fused_gather: 0 runs moe_permute and hands b->xp to the GEMM.  1 (bf16
 *     weights, where the GEMM takes its operand-swapped kernel: at least 16
 *     rows per expert on average, or y_dtype MOE_E4M3) skips the permuted
 *     copy: the gate/up GEMM reads routed row s from row pair_of_slot[s] / k
 *     of a token-major source, x itself for a bf16 payload, or for an FP8
 *     payload each token's round trip bf16(decode(q) * scale) (the rows
 *     moe_permute's payload dequantises to), written once per token into
 *     b->gemm_workspace.  h, y and out are the same; b->xp and b->xp_scales
 *     are not written.  Elsewhere the flag is ignored.
 *     packed_weights: 1 when w13 and w2 hold moe_pack_expert_weights'
 *     output (bf16 weights; the GEMM then runs as moe_grouped_gemm_packed).
 *     weights_in_gemm: 1 (bf16 weights) applies each routed row's router
 *     weight in the down GEMM's epilogue (y row s = topk_w[pair_of_slot[s]]
 *     times the expert's output, fp32 product) and makes the combine a plain
 *     k-way sum in j order (moe_combine with topk_w NULL); out differs from
 *     the default by the rounding of that product (each pick's w*y is
 *     rounded to fp32 before the sum instead of fused into it).
 *     all_reduce_form: 0 runs moe_combine.  1 runs the combine of the
 *     all_reduce form on the W logical ranks: moe_combine_rank for r = 0..W-1
 *     into b->partials[r], then moe_reduce_partials into out (the same sum,
 *     associated by rank).
 *   step_events: NULL, or 8 cudaEvent_t handles recorded on `stream` at:
 *   0 before routing, 1 after routing, 2 after the layout, 3 after the
 *   permute (with fused_gather: after the token-major FP8 round trip, or
 *   at once for a bf16 payload), 4 when the GEMM's bf16 operand is ready
 *   (inside this call an FP8 permute writes it as well, so 4 follows 3
 *   directly), 5 after the
 *   gate/up GEMM, 6 after the down GEMM, 7 after combine -- so that a caller
 *   can time each kernel on the stream it runs on, without launch gaps
 *   between them.
 */
typedef struct moe_layer_options {
    int32_t capacity;          /* -1: dropless; C >= 0: fixed slabs of C rows per expert */
    int32_t route_groups;      /* 0: plain top-k; G: group-limited routing over G groups */
    int32_t route_max_groups;  /* M: groups each token may reach (with route_groups) */
    int32_t fused_gather;      /* 0: permute, then the GEMM; 1: the GEMM gathers the rows */
    int32_t all_reduce_form;   /* 0: one combine; 1: W per-rank partials, then their sum */
    int32_t packed_weights;    /* 0: w13/w2 stacked; 1: in moe_pack_expert_weights' layout */
    int32_t weights_in_gemm;   /* 0: combine weights the rows; 1: the down GEMM does */
} moe_layer_options;

typedef struct moe_layer_buffers {
    int32_t* topk_idx;       /* [T, k] */
    float* topk_w;           /* [T, k] */
    int32_t* expert_counts;  /* [E] */
    int32_t* expert_offsets; /* [E + 1] */
    int32_t* rank_offsets;   /* [W + 1] */
    int32_t* slot_of_pair;   /* [T*k] */
    int32_t* pair_of_slot;   /* [S] slots: S = T*k, or E*capacity */
    void* layout_workspace;  /* moe_dispatch_layout_workspace_bytes(T, k, E) */
    size_t layout_workspace_bytes;
    void* xp;                /* [S, H] payload */
    float* xp_scales;        /* [S, H/128] (FP8 payload only), 16-byte aligned */
    void* h;                 /* [S, I] in w_dtype */
    void* y;                 /* [S, H] in y_dtype */
    float* y_scales;         /* [S, H/128] (FP8 y only) */
    void* gemm_workspace;    /* moe_grouped_gemm_workspace_bytes(S, ...) */
    size_t gemm_workspace_bytes;
    int32_t* dev_status;     /* int32, zero-initialised */
    int32_t* n_dropped;      /* int32 or NULL: dropped pairs (capacity >= 0) */
    float* partials;         /* [W, T, H] fp32 (all_reduce_form only), else NULL */
} moe_layer_buffers;

moe_status moe_layer_forward(const float* logits, const void* x, moe_dtype x_dtype, int64_t T,
                             int32_t H, int32_t E, int32_t k, int32_t W, int32_t I,
                             const void* w13, const void* w2, moe_dtype w_dtype,
                             moe_dtype payload_dtype, moe_dtype y_dtype,
                             const moe_layer_options* opts, const moe_layer_buffers* b, void* out,
                             void* const* step_events, void* stream);

/*
 * moe_layer_forward_host -- moe_layer_forward with the inputs and the
 * output in HOST memory: copies logits and x from the host (cudaMemcpyAsync
 * on `stream`; pinned host memory makes the copies asynchronous), runs the
 * layer, and copies out back to the host.  logits_dev, x_dev and out_dev
 * are device staging buffers of the same shapes.  Returns once everything
 * is enqueued; synchronise the stream before reading out_host.
 */
moe_status moe_layer_forward_host(const float* logits_host, const void* x_host, void* out_host,
                                  float* logits_dev, void* x_dev, void* out_dev,
                                  moe_dtype x_dtype, int64_t T, int32_t H, int32_t E, int32_t k,
                                  int32_t W, int32_t I, const void* w13, const void* w2,
                                  moe_dtype w_dtype, moe_dtype payload_dtype, moe_dtype y_dtype,
                                  const moe_layer_options* opts, const moe_layer_buffers* b,
                                  void* const* step_events, void* stream);

/*
 * moe_check_status -- synchronise `stream`, read the device status word,
 * clear it, and map it to a status: MOE_ERR_TIMEOUT if a wait ran out,
 * else MOE_ERR_OVERFLOW if a row missed a receive buffer, else
 * MOE_ERR_BAD_INDEX if an id was skipped, else MOE_OK (MOE_ERR_CUDA if the
 * synchronisation itself failed).  The only call that blocks.
 */
moe_status moe_check_status(int32_t* dev_status, void* stream);

/* Static, human-readable name of a status code. */
const char* moe_status_str(moe_status s);

/* Diagnostics: total number of kernels this library has launched in this
 * process (all devices, all streams), counted on the host at launch. */
uint64_t moe_launch_count(void);

/*
 * moe_diag_gemm_clock -- diagnostics: the SM clock the operand-swapped
 * grouped GEMM ran at (the bf16 tensor-core kernel moe_grouped_gemm and the
 * layer use from 16 routed rows per expert on average, or with an FP8 y,
 * packed weights or router weights in the GEMM; below that, the token-major
 * kernel runs and records nothing).  Every launch adds, for CTA 0, the SM cycles (clock64) and the
 * nanoseconds (globaltimer) from its first instruction to its last into a
 * per-device record: out[0], out[1] for the gate/up phase, out[2], out[3]
 * for the down phase; cycles / ns is the mean clock in GHz.  Synchronises
 * the current device, then copies the record to out (4 uint64, host; may be
 * NULL) and, with reset non-zero, clears it.  MOE_ERR_CUDA if a copy fails.
 */
moe_status moe_diag_gemm_clock(uint64_t* out, int32_t reset);

/*
 * moe_diag_layout_wait_timeout -- diagnostics for failure detection: runs
 * the dispatch layout's scan kernel (the one moe_dispatch_layout launches)
 * on a two-chunk look-back state in which the first chunk never publishes
 * its count, so the second chunk's bounded wait on that flag can only run
 * out.  After wait_limit_ns of device time (globaltimer) the kernel gives up,
 * OR-s MOE_DEV_TIMEOUT into dev_status and returns; moe_check_status then
 * reports MOE_ERR_TIMEOUT.  Nothing faults, traps or hangs, and the context
 * stays usable.  The library's own calls bound this wait at 2 s; here the
 * limit is the caller's, at most 2 s (MOE_ERR_INVALID_ARG above that).
 *
 *   workspace  device scratch of moe_diag_layout_wait_timeout_workspace_bytes()
 *              bytes, 16-byte aligned, clobbered.
 *   dev_status int32 device word.
 */
size_t moe_diag_layout_wait_timeout_workspace_bytes(void);
moe_status moe_diag_layout_wait_timeout(void* workspace, size_t workspace_bytes,
                                        uint64_t wait_limit_ns, int32_t* dev_status,
                                        void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
