/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE-layer forward library (libmoe_b200.so).
 *
 * The library computes the forward pass of a token-choice top-k Mixture-of-Experts
 * layer on one GPU, one stream-ordered step per call:
 *
 *   moe_prepare_router_weight  the router's exact bf16 split of W_g, once at load time
 *   moe_route            router logits (fp32), scoring, optional selection-only bias,
 *                        top-k, renormalised and scaled gates
 *   moe_histogram_scan   per-expert counts, capacity clamp, token-order ranks,
 *                        expert-contiguous row offsets and the row maps
 *   moe_permute          gather tokens into expert-contiguous rows
 *   moe_expert_gate_up   grouped GEMM  H = silu(X Wg^T) * (X Wu^T)       (per expert)
 *   moe_expert_gate_up_gather  the same with the permute fused into it (X read via the row map)
 *   moe_expert_down      grouped GEMM  Y = gate_of_row * (H Wd^T)       (per expert)
 *   moe_grouped_ffn      the two GEMMs above back to back
 *   moe_combine          gate-weighted sum of each token's rows (+ shared expert)
 *   moe_expert_down_combine  the down GEMM with the combine fused into its epilogue
 *   moe_expert_gate_up_fp4 / moe_expert_down_fp4  the expert GEMMs with 4-bit weights
 *   moe_round_output     the combine's final rounding of an fp32 sum to bf16
 *   moe_router_stats     per-expert load, aux loss, z-loss, drops, imbalance
 *
 * Sources (web pages on Mixture-of-Experts, cited by title and section):
 *   [MoE-Explained]  "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡"
 *                    (Chinese rendering of Hugging Face's "Mixture of Experts Explained")
 *   [Handbook-News]  "Hugging Face 团队投入 ~80 万 GPU 小时…「终极 MoE 训练手册」" (hub.geekagi.cn)
 *   [Handbook-Digest] "Hugging Face 发布 3 万词免费 MoE 训练手册" (agihunt.info)
 *   [Handbook-Article] "Hugging Face开源MoE训练手册：基于80万GH200卡时沉淀Megatron-LM实战" (zicq.com)
 *
 * Conventions for every call
 *   - Pointers marked (device) must point to device memory owned by the caller, and
 *     pointers marked (host) to host memory; the library allocates nothing and keeps no
 *     state except one device error word (and the fixed scratch array of
 *     moe_histogram_scan_noalloc).
 *   - All launches are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No call synchronises the host, except moe_get_device_error.
 *   - Layouts are dense row-major (C order) with the leading dimension equal to the
 *     row length.  bf16 = IEEE bfloat16 stored in 2 bytes.
 *   - Arguments are validated on the host before any launch; a failed check returns
 *     MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE and launches nothing.
 *     A launch error returns MOE_ERR_CUDA (moe_last_cuda_error() names it).
 *   - Corrupt device data (an expert id outside [0,E), a token naming one expert twice,
 *     a bounded wait that gave up) never traps: the kernel records a MOE_DEVERR_* code
 *     in the device error word, skips the bad access and finishes; read it with
 *     moe_get_device_error.
 *   - Supported sizes: 1 <= E <= 1024, 1 <= k <= min(E, 32), 0 <= T < 2^24,
 *     d % 8 == 0, F % 8 == 0 (16-byte row strides), device pointers 16-byte aligned.
 *
 * Numerical contract
 *   - Router logits are fp32 sums of fp32(x) * Wg (bf16 x is widened exactly).
 *   - Top-k selects by the logit (no selection bias) or by score + bias evaluated in
 *     fp64 (with a selection bias); ties go to the lower expert index; outputs are
 *     ordered by key descending, then index ascending.
 *   - Routing indices, counts, offsets and row maps are exact integers and
 *     deterministic run to run.
 *   - Expert GEMMs take bf16 operands with fp32 accumulation; H is rounded to bf16
 *     (round to nearest even) because it is the down GEMM's tensor-core operand.  The
 *     gated expert rows and the layer output are written in the dtype the caller picks
 *     (fp32 keeps H as the only rounding inside the layer; bf16 rounds each row and the
 *     output once more).  The combine sums in fp32 in slot order j = 0..k-1, then adds
 *     the shared expert, then converts to the output dtype.  moe_expert_down_combine
 *     adds the same fp32 terms in the order its tiles finish instead (not bitwise
 *     reproducible; each result is within fp32 rounding of the ordered sum).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

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

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, negative size, k > E, unknown enum, ...   */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but outside the supported sizes / alignments      */
  MOE_ERR_WORKSPACE = 3,    /* workspace pointer null or smaller than the query result */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed                       */
  MOE_ERR_DEVICE = 5        /* moe_get_device_error found a recorded device error      */
} moe_status;

typedef enum {
  MOE_SCORE_SOFTMAX = 0,        /* softmax over experts                 */
  MOE_SCORE_SIGMOID = 1,        /* 1 / (1 + e^-l) per expert            */
  MOE_SCORE_SQRT_SOFTPLUS = 2   /* sqrt(log(1 + e^l)) per expert        */
} moe_score;

typedef enum { MOE_BF16 = 0, MOE_F32 = 1 } moe_dtype;

typedef enum {
  MOE_FP4_MX = 0,               /* MXFP4: 32-element blocks, E8M0 power-of-two scales      */
  MOE_FP4_NV = 1                /* NVFP4: 16-element blocks, E4M3 scales + an fp32 scale   */
} moe_fp4_format;

typedef enum {
  MOE_SELECT_UNIFORM = 0,       /* slot j of token t takes expert (t k + j) mod E        */
  MOE_SELECT_HASH = 1           /* k distinct experts from a hash of the token id         */
} moe_select_rule;

/* Device error codes recorded by kernels (first one wins until read). */
#define MOE_DEVERR_NONE 0
#define MOE_DEVERR_EXPERT_ID 1      /* a topk_idx entry outside [0, E)                   */
#define MOE_DEVERR_DUP_EXPERT 2     /* one token lists the same expert twice             */
#define MOE_DEVERR_ROW 3            /* a row index outside its buffer                    */
#define MOE_DEVERR_SCAN_TIMEOUT 4   /* scan look-back wait gave up (bounded spin)        */
#define MOE_DEVERR_PIPE_TIMEOUT 5   /* GEMM pipeline barrier wait gave up (bounded spin) */

/* ------------------------------------------------------------------------------------
 * moe_capacity -- expert capacity in slots.
 * [MoE-Explained] section "Switch Transformer", eq. Expert Capacity =
 * (tokens per batch / number of experts) x capacity factor; the overflow rule is in
 * section "MoE 与 Transformer".
 *   per_assignment != 0: ceil(cf * T * k / E)   (tokens per batch counted as T*k)
 *   per_assignment == 0: ceil(cf * T / E)       (the literal top-1 form)
 * Evaluated in double.  Returns -1 (no dropping) when cf <= 0, and -2 for T < 0,
 * E < 1 or k < 1.
 * ---------------------------------------------------------------------------------- */
MOE_API int32_t moe_capacity(int32_t T, int32_t E, int32_t k, double capacity_factor,
                     int32_t per_assignment);

/* Rows the permuted buffers must hold: T*k when capacity < 0, else min(T*k, E*capacity). */
MOE_API int64_t moe_rows_max(int32_t T, int32_t E, int32_t k, int32_t capacity);

/* Which tile orientation the bf16 gate/up GEMMs (moe_expert_gate_up and
 * moe_expert_gate_up_gather) take for these sizes: 1 = weight-major (256 weight rows x
 * an expert's tokens; chosen when the groups average under 1024 rows, rows_max / E), 0 =
 * token-major (256 token rows of one expert x 256 outputs).  The environment variable
 * MOE_B200_EXPERT_TILES=tokens|weights overrides the choice, here as in the GEMMs.  A
 * caller can use it to pick its dispatch form: the gathered gate/up reads x through
 * token_of_row at no extra cost in the weight-major orientation (the token rows are the
 * small operand), while the token-major one re-reads each row once per output tile.
 * Returns -1 for rows_max < 0 or E < 1.  Host only. */
MOE_API int32_t moe_gate_up_weight_major(int64_t rows_max, int32_t E);

/* ------------------------------------------------------------------------------------
 * moe_prepare_router_weight -- the tensor-core router's operand, made once at load time.
 * [MoE-Explained] section "Switch Transformer" (the router stays in full precision);
 * [Handbook-News] "真正难在三个环节" item 1 (FP32 routing).
 * The router multiplies a bf16 x by an fp32 W_g on bf16 tensor cores by splitting W_g
 * exactly into three bf16 terms, hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi -
 * mid): the three carry all 24 significant bits of w, every product x * term is exact
 * in fp32, and the MMAs accumulate in fp32, so the logits are fp32 sums of the exact
 * products x . W_g.  This call writes that split for a given W_g; W_g does not change
 * between forwards, so do it once (and again whenever W_g changes) and pass the result
 * to moe_route / moe_router_logits.
 *   Wg          (device) [d, E] fp32
 *   Wg_split    (device) out, moe_router_weight_bytes(d, E) bytes, 16-byte aligned,
 *               owned by the caller.  Layout: experts in n = ceil(E / 256) tiles of
 *               NE = 32 * ceil(ceil(E / n) / 32) experts; tile j holds, as rows of a
 *               K-major bf16 matrix [3 n NE, d], the hi terms of experts j NE .. j NE +
 *               NE - 1, then their mid terms, then their lo terms (zero past E).
 * moe_router_weight_bytes returns 0 when the tensor-core router does not apply to (d, E)
 * (d < 64, d % 8 != 0, E % 4 != 0 or E > 1024); moe_prepare_router_weight then returns
 * MOE_ERR_UNSUPPORTED and the router reads W_g directly.
 * Errors: INVALID_ARG for a null pointer, d < 1 or E < 1; UNSUPPORTED as above or for an
 * unaligned Wg_split; WORKSPACE when bytes is below the query.
 * ---------------------------------------------------------------------------------- */
MOE_API size_t moe_router_weight_bytes(int32_t d, int32_t E);
MOE_API moe_status moe_prepare_router_weight(const float* Wg, int32_t d, int32_t E, void* Wg_split,
                     size_t bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_route -- router, scoring, top-k and gates.
 * [MoE-Explained] section "什么是稀疏性？": G_sigma(x) = Softmax(x . W_g),
 * KeepTopK(v, k), G(x) = Softmax(KeepTopK(H(x), k)); section "Switch Transformer"
 * (router kept in full precision); [Handbook-News] "真正难在三个环节" item 1 (FP32
 * routing) and item 2 (loss-free bias), tweet (softmax / sigmoid / sqrt(softplus));
 * [Handbook-Digest] "已确认" (sqrt(softplus) scoring, scale factor near sqrt(k)).
 *
 *   x            (device) [T, d], x_dtype (MOE_BF16 or MOE_F32)
 *   Wg           (device) [d, E] fp32
 *   Wg_split     (device) the result of moe_prepare_router_weight for this Wg, or NULL:
 *                the call then splits W_g itself, into the workspace (one more launch)
 *   logit_offset (device) [E] fp32 or NULL: added to every logit (enters selection and gates)
 *   select_bias  (device) [E] fp32 or NULL: added to the score for selection only
 *   score        moe_score;  renormalize 0/1;  scale multiplies the final gates
 *   logits       (device) [T, E] fp32 out: x . Wg + logit_offset
 *   topk_idx     (device) [T, k] int32 out
 *   topk_gate    (device) [T, k] fp32 out
 *   workspace    (device) >= moe_route_workspace_bytes(T, d, E) bytes (may be NULL if 0);
 *                the query covers every call with at most T tokens (same d, E), with or
 *                without a prepared weight
 * Paths: bf16 x with T >= 256, d >= 64 and E % 4 == 0 runs one tensor-core kernel (CTA
 * pairs, 256 tokens per tile) that also selects the top-k and computes the gates in its
 * epilogue (softmax scores with a selection bias add a separate top-k pass: their keys
 * need the whole row's normaliser first).  Otherwise an fp32 SIMT GEMM and a top-k
 * kernel run.
 * Gates: softmax + renormalize -> softmax over the k kept logits; softmax without
 * renormalize -> the full softmax probability; sigmoid / sqrt(softplus) -> kept scores
 * over their sum (renormalize) or the scores; all then times scale.  The softmax over
 * the kept logits takes each difference to their maximum and its exponential in fp64,
 * then rounds the gate to fp32 (the same for moe_route_fixed and moe_route_noisy).
 * ---------------------------------------------------------------------------------- */
MOE_API size_t moe_route_workspace_bytes(int32_t T, int32_t d, int32_t E);
MOE_API moe_status moe_route(const void* x, int32_t x_dtype, const float* Wg, const void* Wg_split,
                     const float* logit_offset, const float* select_bias,
                     int32_t T, int32_t d, int32_t E, int32_t k,
                     int32_t score, int32_t renormalize, float scale,
                     float* logits, int32_t* topk_idx, float* topk_gate,
                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_router_logits -- the router alone: logits = x . Wg (+ logit_offset), fp32.
 * [MoE-Explained] section "什么是稀疏性？" (x . W_g); section "Switch Transformer"
 * (router in full precision); [Handbook-News] "真正难在三个环节" item 1 (FP32 routing).
 * The same GEMM as moe_route (bf16 x with T >= 256, d >= 64 and E % 4 == 0: tensor
 * cores over the three-term split of W_g; otherwise fp32 SIMT), without the top-k.  It
 * also gives the noise logits x . W_noise of moe_route_noisy.
 *   x            (device) [T, d], x_dtype;  16-byte aligned
 *   Wg           (device) [d, E] fp32
 *   Wg_split     (device) moe_prepare_router_weight's result for this Wg, or NULL (split
 *                into the workspace by the call)
 *   logit_offset (device) [E] fp32 or NULL
 *   logits       (device) [T, E] fp32 out
 *   workspace    (device) >= moe_router_logits_workspace_bytes(T, d, E) bytes (may be
 *                NULL if 0)
 * Errors: INVALID_ARG for a null pointer, T < 0, E < 1 or an unknown dtype;
 * UNSUPPORTED for E > 1024, d % 8 != 0 or an unaligned x or Wg_split; WORKSPACE if too
 * small.
 * ---------------------------------------------------------------------------------- */
MOE_API size_t moe_router_logits_workspace_bytes(int32_t T, int32_t d, int32_t E);
MOE_API moe_status moe_router_logits(const void* x, int32_t x_dtype, const float* Wg, const void* Wg_split,
                     const float* logit_offset, int32_t T, int32_t d, int32_t E,
                     float* logits, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_route_fixed -- a fixed selection rule with the learned router's gates.
 * MOE_SELECT_UNIFORM: [Handbook-News] "真正难在三个环节" item 2 (a control run with
 *   routing forced uniform was about 1.5x faster: the speed headroom of balance).  Slot
 *   j of token t takes expert (t k + j) mod E, so every expert receives floor(T k / E)
 *   or ceil(T k / E) assignments.
 * MOE_SELECT_HASH: [Handbook-Digest] "已确认" (DeepSeek-V4's first three MoE layers
 *   choose experts by a fixed hash of the token id).  Floyd's sampling of k distinct
 *   experts: with base = fmix32(token_id[t] ^ seed) (fmix32 = MurmurHash3's 32-bit
 *   finalizer) and, for j = 0 .. k-1, n = E - k + j and r = fmix32(base + j) mod (n + 1),
 *   slot j takes r unless an earlier slot holds it, else n.  Same id, same experts.
 *   logits      (device) [T, E] fp32: the router logits (moe_router_logits)
 *   score, renormalize, scale: as moe_route; the gates of the chosen experts follow
 *               moe_route's rule (softmax over the chosen logits, the full softmax
 *               probability, or the chosen scores over their sum / the scores) x scale
 *   rule        moe_select_rule
 *   token_id    (device) [T] int32 for MOE_SELECT_HASH (any value), else may be NULL
 *   seed        mixed into the hash
 *   topk_idx    (device) [T, k] int32 out, in slot order (not sorted)
 *   topk_gate   (device) [T, k] fp32 out
 * Errors: INVALID_ARG for a null pointer, T < 0, k < 1, k > E, an unknown score or rule,
 * renormalize not 0/1 or a non-finite scale; UNSUPPORTED for E > 1024 or k > 32.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_route_fixed(const float* logits, int32_t T, int32_t E, int32_t k,
                     int32_t score, int32_t renormalize, float scale, int32_t rule,
                     const int32_t* token_id, uint32_t seed, int32_t* topk_idx,
                     float* topk_gate, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_route_noisy -- noisy top-k gating.
 * [MoE-Explained] section "什么是稀疏性？": H(x)_i = (x . W_g)_i + StandardNormal() *
 * Softplus((x . W_noise)_i); G(x) = Softmax(KeepTopK(H(x), k)).
 *   logits       (device) [T, E] fp32: x . W_g (+ offset)
 *   logits_noise (device) [T, E] fp32: x . W_noise (moe_router_logits with W_noise)
 *   noise        (device) [T, E] fp32: the standard normal draws, supplied by the caller
 *   scale        multiplies the gates
 *   H            (device) [T, E] fp32 out: l + n * softplus(l_noise) in fp32, softplus
 *                as max(z, 0) + log1p(exp(-|z|)), one rounding for the product and sum;
 *                must not overlap the inputs
 *   topk_idx     (device) [T, k] int32 out: the k largest H, ties to the lower index,
 *                order H descending then index ascending
 *   topk_gate    (device) [T, k] fp32 out: softmax over the kept H, x scale
 * Errors: INVALID_ARG for a null pointer, T < 0, k < 1, k > E or a non-finite scale;
 * UNSUPPORTED for E > 1024 or k > 32.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_route_noisy(const float* logits, const float* logits_noise,
                     const float* noise, int32_t T, int32_t E, int32_t k, float scale,
                     float* H, int32_t* topk_idx, float* topk_gate, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_histogram_scan -- counts, capacity, token-order ranks, offsets, row maps.
 * [MoE-Explained] section "MoE 与 Transformer" (an expert takes at most `capacity`
 * tokens; overflow leaves through the residual or is dropped) and section
 * "更多关于高效训练的内容" (uneven groups, no padding); [Handbook-Article] (capacity
 * limit, overflow tokens dropped).
 *
 *   topk_idx, topk_gate (device) [T, k]: a token's k experts must be distinct
 *   capacity     slots per expert, or -1 for no dropping
 *   counts       (device) [E] int32 out: assignments per expert before dropping
 *   kept         (device) [E] int32 out: min(counts, capacity)
 *   offsets      (device) [E+1] int32 out: exclusive scan of kept; offsets[E] = rows used
 *   row_of       (device) [T, k] int32 out: row of assignment (t, j), or -1 if dropped
 *   token_of_row (device) [rows_max] int32 out: token of each used row
 *   gate_of_row  (device) [rows_max] fp32 out: gate of each used row
 *   workspace    (device) >= moe_histogram_scan_workspace_bytes(T, k, E) bytes; the
 *                call clears what it needs (one memset node on `stream`).
 * rank(t, j) = number of tokens t' < t whose top-k holds expert idx[t, j]; the
 * assignment is kept iff rank < capacity; row_of = offsets[e] + rank.  Rows inside an
 * expert are in token order.  Entries of token_of_row / gate_of_row at rows >=
 * offsets[E] are left untouched.
 * ---------------------------------------------------------------------------------- */
MOE_API size_t moe_histogram_scan_workspace_bytes(int32_t T, int32_t k, int32_t E);
MOE_API moe_status moe_histogram_scan(const int32_t* topk_idx, const float* topk_gate,
                              int32_t T, int32_t k, int32_t E, int32_t capacity,
                              int32_t* counts, int32_t* kept, int32_t* offsets,
                              int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Expert-parallel forward (one process per GPU, G ranks): the per-rank building blocks.
 * [MoE-Explained] section "让 MoE 起飞" / expert parallelism (experts on different
 * workers; tokens are sent to the workers holding their experts and the results sent
 * back) and section "Switch Transformer" (expert capacity); [Handbook-News] "真正难在三个
 * 环节" item 3 (the dispatch / combine all-to-all of every MoE layer).
 * Rank h owns experts [h E/G, (h+1) E/G) (E % G == 0).  The global token order is rank
 * 0's tokens, then rank 1's, ...; capacity drops follow it.  A rank's forward:
 *   moe_route (all E experts) -> moe_histogram_scan (capacity -1: the local counts) ->
 *   all-gather the counts [G][E] -> moe_ep_plan_host -> moe_histogram_scan_caps (the
 *   rank's kept limit per expert) -> moe_permute (rows grouped by expert, so by
 *   destination) -> all-to-all (send_rows / recv_rows) -> moe_ep_regroup (source-major to
 *   expert-major) -> the grouped GEMMs over the local experts (no gate) ->
 *   moe_ep_regroup inverse -> all-to-all back -> moe_combine with topk_gate.
 *
 * moe_histogram_scan_caps -- moe_histogram_scan with a per-expert capacity: expert e keeps
 *   its first caps[e] assignments in token order (caps: device [E] int32).  The row
 *   buffers hold T*k rows.  Other arguments, workspace and errors as moe_histogram_scan.
 *
 * moe_ep_plan_host -- the dispatch plan of rank g, on the host.
 *   counts        (host) [G][E] int32: every rank's per-expert assignment counts
 *   capacity      slots per expert for the whole batch, or -1 (no dropping)
 *   caps          (host) [E] out: kept[g][e] = clamp(capacity - sum_{s<g} counts[s][e], 0,
 *                 counts[g][e]) (counts[g][e] without a capacity)
 *   send_rows     (host) [G] out: rows rank g sends to each rank (its kept rows of that
 *                 rank's experts)
 *   recv_rows     (host) [G] out: rows each rank sends to rank g
 *   local_offsets (host) [E/G + 1] out: rank g's experts' rows, expert by expert (sources
 *                 in rank order inside an expert), as a grouped GEMM's offsets
 *   regroup       (host) [G * E/G][3] int64 out: for source s and local expert j, entry
 *                 s E/G + j = (row in the receive buffer, row in the expert-major buffer,
 *                 rows)
 *   Errors: INVALID_ARG for G < 1, g outside [0, G), negative counts, a null pointer or
 *   capacity < -1; UNSUPPORTED for E % G != 0 or E > 1024.
 *
 * moe_ep_regroup -- row copies by a regroup table (device [n][3] int64, as written by
 *   moe_ep_plan_host): inverse 0 copies src row (entry[0] + r) to dst row (entry[1] + r),
 *   inverse 1 the other way; rows of row_bytes bytes (a multiple of 16).  An entry that
 *   would leave either buffer records MOE_DEVERR_ROW and is skipped.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_histogram_scan_caps(const int32_t* topk_idx, const float* topk_gate,
                              int32_t T, int32_t k, int32_t E, const int32_t* caps,
                              int32_t* counts, int32_t* kept, int32_t* offsets,
                              int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                              void* workspace, size_t workspace_bytes, void* stream);
MOE_API moe_status moe_ep_plan_host(const int32_t* counts, int32_t G, int32_t g, int32_t E,
                              int32_t capacity, int32_t* caps, int64_t* send_rows,
                              int64_t* recv_rows, int32_t* local_offsets, int64_t* regroup);
MOE_API moe_status moe_ep_regroup(const void* src, int64_t src_rows, int32_t row_bytes,
                              const int64_t* table, int32_t n, int32_t inverse, void* dst,
                              int64_t dst_rows, void* stream);

/* ------------------------------------------------------------------------------------
 * The expert-parallel exchange fused into the dispatch and the combine, over peer memory.
 * [MoE-Explained] section "让 MoE 起飞" (expert parallelism); [Handbook-News]
 * "真正难在三个环节" item 3 (the dispatch and combine all-to-all is where the time goes).
 * Each rank holds, for every owner h (itself included), a device pointer to h's
 * expert-major row buffer (peer_rows, device [G] array of pointers: peers' memory mapped
 * by moe_ipc_open_handle, or this GPU's own buffer) and its capacity in rows
 * (peer_rows_cap, device [G] int64).  The owner's rows of its experts are laid out exactly
 * as moe_ep_plan_host's local_offsets say (expert by expert, source ranks in order inside
 * an expert), so a source can write each of its kept rows straight to its final place:
 *   moe_route -> moe_histogram_scan (-1) -> all-gather counts -> moe_ep_plan_host (caps,
 *   local_offsets) and moe_ep_dst_base_host (dst_base) -> moe_histogram_scan_caps ->
 *   moe_ep_dispatch (x rows -> owners' buffers) -> a barrier of the G ranks -> the grouped
 *   GEMMs over the local rows (no gate) -> a barrier -> moe_ep_combine (owners' result
 *   rows -> y, with topk_gate).
 * This replaces moe_permute, both all-to-alls, both regroupings and moe_combine.  The
 * barriers are the caller's (a stream-ordered collective of the process group): no kernel
 * here waits on another GPU.  No load uses cluster multicast.
 *
 * moe_ep_dst_base_host -- for rank g's kept rows of expert e, their first row in the
 *   owner's buffer: local_offsets_owner[e mod E/G] + the rows of e kept by ranks before g.
 *   counts (host) [G][E] int32, capacity as moe_ep_plan_host; dst_base (host) [E] out.
 *   Errors as moe_ep_plan_host.
 *
 * moe_ep_dispatch -- x [T, d] (bf16 or fp32, dtype) of this rank; topk_idx, row_of [T, k]
 *   and offsets [E+1] from moe_histogram_scan_caps (row_of indexes this rank's expert-major
 *   rows, rows_max of them; offsets are this rank's); dst_base (device) [E] int32 from
 *   moe_ep_dst_base_host.  Stores x[t] into peer_rows[e / (E/G)] at row dst_base[e] +
 *   (row_of[t][j] - offsets[e]) for each kept slot j of expert e = topk_idx[t][j].  A slot
 *   whose row is not expert e's, whose expert is out of range or whose position is past
 *   the owner's capacity records MOE_DEVERR_ROW and is skipped; a null owner pointer is
 *   skipped.  d * element size a multiple of 16; x 16-byte aligned.
 *   Errors: INVALID_ARG for bad sizes or dtypes, E % G != 0 or a null pointer (T > 0);
 *   UNSUPPORTED for a row size that is not a multiple of 16 bytes or a misaligned x.
 *
 * moe_ep_combine -- y [T, d] (y_dtype) = sum over the kept slots j, in slot order, of
 *   topk_gate[t][j] * (the owner's row of that slot, rows_dtype), in fp32, rounded once;
 *   tokens with no kept slot get zeros.  The rows are found as in moe_ep_dispatch, in
 *   peer_rows (the owners' down-GEMM outputs, ungated).  The same sum as moe_combine with
 *   topk_gate over those rows.  Errors as moe_ep_dispatch (d a multiple of 8, y 16-byte
 *   aligned).
 *
 * moe_ipc_handle_bytes -- the size of a handle (64).
 * moe_ipc_get_handle -- the CUDA IPC handle of the allocation holding the device pointer
 *   ptr, and ptr's offset in it (handle: host, moe_ipc_handle_bytes bytes; offset: host).
 * moe_ipc_open_handle -- maps another process's allocation into this one (peer access
 *   enabled): *base is the mapping, *ptr = *base + offset.  Close with moe_ipc_close(base).
 *   A handle from this same process cannot be opened (CUDA refuses it): a rank uses its
 *   own pointer for itself.
 * Errors: INVALID_ARG for null pointers or a pointer CUDA does not know; UNSUPPORTED when
 * the driver entry point is missing; CUDA for a refused mapping.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_ep_dst_base_host(const int32_t* counts, int32_t G, int32_t g, int32_t E,
                              int32_t capacity, int32_t* dst_base);
MOE_API moe_status moe_ep_dispatch(const void* x, int32_t dtype, int32_t T, int32_t d, int32_t k,
                              const int32_t* topk_idx, const int32_t* row_of,
                              const int32_t* offsets, const int32_t* dst_base, int32_t E,
                              int32_t G, int64_t rows_max, const void* const* peer_rows,
                              const int64_t* peer_rows_cap, void* stream);
MOE_API moe_status moe_ep_combine(const void* const* peer_rows, int32_t rows_dtype,
                              const int64_t* peer_rows_cap, int32_t G, const int32_t* topk_idx,
                              const int32_t* row_of, const float* topk_gate,
                              const int32_t* offsets, const int32_t* dst_base, int32_t E,
                              int32_t T, int32_t d, int32_t k, int64_t rows_max,
                              int32_t y_dtype, void* y, void* stream);
MOE_API int32_t moe_ipc_handle_bytes(void);
MOE_API moe_status moe_ipc_get_handle(const void* ptr, void* handle, int64_t* offset);
MOE_API moe_status moe_ipc_open_handle(const void* handle, int64_t offset, void** ptr, void** base);
MOE_API moe_status moe_ipc_close(void* base);

/* ------------------------------------------------------------------------------------
 * moe_scan_wait_check -- diagnostic: makes the histogram/scan's bounded wait run out.
 * (No counterpart on the pages: it tests the library's own recovery path.)
 * The look-back of moe_histogram_scan's rank kernel waits for the running totals of the
 * chunks of 256 tokens before it; every such wait is bounded.  This call runs the same
 * kernels with the first chunk withheld, so every later chunk waits for a word that is
 * never published.  Each wait gives up after wait_ns nanoseconds, records
 * MOE_DEVERR_SCAN_TIMEOUT in the device error word and lets the kernel finish; the
 * call returns MOE_OK once launched, and the context stays usable.  Nothing traps or
 * faults: every index stays bounded whatever the totals.  The outputs are not meaningful.
 *   arguments as moe_histogram_scan, plus
 *   wait_ns      1e3 .. 1e9: the per-wait limit (the ordinary calls use one second)
 * Errors: INVALID_ARG for T <= 256 (there must be a chunk after the first), a null
 * pointer or wait_ns outside its range; WORKSPACE as moe_histogram_scan.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_scan_wait_check(const int32_t* topk_idx, const float* topk_gate,
                              int32_t T, int32_t k, int32_t E, int32_t capacity,
                              int32_t* counts, int32_t* kept, int32_t* offsets,
                              int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                              uint64_t wait_ns, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_histogram_scan_noalloc -- moe_histogram_scan for callers that cannot allocate.
 * (No counterpart on the pages: this is a deployment convenience, not part of the method.)
 *
 * Some callers may not allocate device memory once they run: a serving runtime that
 * reserves all of its memory at start-up and forbids later cudaMalloc, a plugin hosted
 * by another framework that hands it no workspace, or a latency-critical loop that
 * cannot afford cudaMalloc's implicit device synchronisation.  This entry point takes
 * the same arguments as moe_histogram_scan minus the workspace, and uses instead a
 * scratch array that the library itself holds in device memory: 4 MiB, a static
 * __device__ array that every GPU using the library keeps until the process exits.
 *
 *   - Limit: moe_histogram_scan_workspace_bytes(T, k, E) must be <= 4 MiB (4194304);
 *     larger sizes return MOE_ERR_WORKSPACE without launching anything (this check comes
 *     before the pointer checks).  The handbook workload (T=8192, k=8, E=64) needs about
 *     0.3 MiB, T=32768 k=16 E=896 about 2.5 MiB.
 *   - The kernels run on the CURRENT device and use that device's copy of the array: the
 *     buffers must live on the current device.  Device ordinals 64 and above return
 *     MOE_ERR_UNSUPPORTED.
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current); make that first call before any stream capture.  The
 *     address is kept for the life of the process: after cudaDeviceReset the library
 *     must be unloaded and loaded again.
 *   - The call allocates nothing: it clears the part of the array that must start at
 *     zero with one memset node on `stream`, then launches the same kernels.
 *   - Every call shares the one array, which keeps the previous call's contents.  Calls
 *     that overlap on the GPU (on different streams, or from several threads without
 *     ordering) race on it and produce wrong results; order them on one stream.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_histogram_scan_noalloc(const int32_t* topk_idx, const float* topk_gate,
                              int32_t T, int32_t k, int32_t E, int32_t capacity,
                              int32_t* counts, int32_t* kept, int32_t* offsets,
                              int32_t* row_of, int32_t* token_of_row, float* gate_of_row,
                              void* stream);

/* ------------------------------------------------------------------------------------
 * moe_permute -- x_perm[row_of[t, j]] = x[t] for every kept assignment.
 * "Send each token to its experts" ([Handbook-News] "MoE 到底省了什么";
 * [Handbook-Article] dispatch as the real bottleneck).
 *   x       (device) [T, d] dtype;   row_of (device) [T, k]
 *   x_perm  (device) [rows_max, d] dtype out (rows >= offsets[E] untouched)
 *   A row index >= rows_max is skipped and recorded as MOE_DEVERR_ROW.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_permute(const void* x, int32_t dtype, int32_t T, int32_t d, int32_t k,
                       const int32_t* row_of, int64_t rows_max, void* x_perm, void* stream);

/* ------------------------------------------------------------------------------------
 * Expert FFN, SwiGLU per expert over expert-contiguous rows.
 * [MoE-Explained] section "什么是混合专家模型": each expert is an FFN; section
 * "更多关于高效训练的内容": uneven token counts per expert handled without padding.
 *
 *   x_rows   (device) [rows_max, d] dtype: rows [offsets[e], offsets[e+1]) belong to e
 *   offsets  (device) [E+1] int32 (non-decreasing, offsets[0] = 0, offsets[E] <= rows_max)
 *   W_gu     (device) [E, 2F, d] dtype: rows 0..F-1 = W_gate[e], rows F..2F-1 = W_up[e]
 *   W_dn     (device) [E, d, F] dtype
 *   h        (device) [rows_max, F] dtype: H = silu(x W_gate^T) * (x W_up^T)
 *   gate_of_row (device) [rows_max] fp32 or NULL (NULL = weight 1, e.g. a shared expert)
 *   y_dtype  dtype of y_rows (MOE_F32 or MOE_BF16; any dtype may be paired with any y_dtype)
 *   y_rows   (device) [rows_max, d] y_dtype out: gate_of_row * (H W_dn^T)
 * bf16 uses the tcgen05 tensor-core path; fp32 uses an fp32 SIMT path.  Rows at or
 * beyond offsets[E] are neither read into results nor written.
 * A shared expert is the call with E = 1, offsets = {0, T} and x_rows = x.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_expert_gate_up(const void* x_rows, int32_t dtype, const int32_t* offsets,
                              int32_t E, int32_t d, int32_t F, int64_t rows_max,
                              const void* W_gu, void* h, void* stream);
/* moe_expert_gate_up_gather -- moe_expert_gate_up with the dispatch fused into it: row r
 * of the GEMM's A operand is read from x[token_of_row[r]] directly ([Handbook-News]
 * "MoE 到底省了什么": sending each token to its experts), so the permuted copy x_perm is
 * neither written nor read and moe_permute is not needed before it.
 *   x (device) [T, d] dtype;  token_of_row (device) [rows_max] int32 from
 *   moe_histogram_scan;  the other arguments as moe_expert_gate_up.
 * Weight-major tiles fetch the rows by TMA row gathers (four rows per instruction),
 * token-major tiles by 16-byte cp.async.  H is bitwise identical to moe_permute followed
 * by moe_expert_gate_up.  A token index outside [0, T) is recorded as MOE_DEVERR_ROW and
 * a row of zeros (token-major) or row 0 of x (weight-major) is read in its place. */
MOE_API moe_status moe_expert_gate_up_gather(const void* x, int32_t dtype, int32_t T,
                              const int32_t* token_of_row, const int32_t* offsets,
                              int32_t E, int32_t d, int32_t F, int64_t rows_max,
                              const void* W_gu, void* h, void* stream);
MOE_API moe_status moe_expert_down(const void* h, int32_t dtype, const int32_t* offsets,
                           int32_t E, int32_t d, int32_t F, int64_t rows_max,
                           const void* W_dn, const float* gate_of_row, int32_t y_dtype,
                           void* y_rows, void* stream);
MOE_API moe_status moe_grouped_ffn(const void* x_rows, int32_t dtype, const int32_t* offsets,
                           int32_t E, int32_t d, int32_t F, int64_t rows_max,
                           const void* W_gu, const void* W_dn, const float* gate_of_row,
                           void* h, int32_t y_dtype, void* y_rows, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_expert_down_combine -- the down projection with the combine fused into it:
 *     y[token_of_row[r]] += gate_of_row[r] * (H[r] W_dn[e]^T)   for every kept row r.
 * The same sum as moe_expert_down followed by moe_combine ([Handbook-News] "MoE 到底
 * 省了什么": gather the experts' results back per token), without writing the gated
 * rows to memory.
 *   h, offsets, W_dn, gate_of_row: as moe_expert_down (gate_of_row NULL = weight 1)
 *   token_of_row (device) [rows_max] int32 from moe_histogram_scan
 *   T        rows of y;   y (device) [T, d] fp32, 16-byte aligned
 *   accumulate 0: y is zeroed first (cudaMemsetAsync on stream);
 *              1: rows are added onto y's contents (e.g. a shared expert's output
 *                 written there by moe_expert_down with E = 1 and y_dtype MOE_F32).
 * Each token's terms are added with fp32 atomics in the order the tiles finish, so y
 * is not bitwise reproducible from run to run (each result is within fp32 rounding of
 * the ordered sum); moe_combine is the reproducible form.  A token index outside
 * [0, T) is skipped and recorded as MOE_DEVERR_ROW.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_expert_down_combine(const void* h, int32_t dtype, const int32_t* offsets,
                           int32_t E, int32_t d, int32_t F, int64_t rows_max,
                           const void* W_dn, const float* gate_of_row,
                           const int32_t* token_of_row, int32_t T, int32_t accumulate,
                           float* y, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_round_output -- y[i] = bf16_rne(y32[i]) for 0 <= i < n: the final rounding of the
 * combine ([MoE-Explained] section "什么是稀疏性？", y = sum_i G(x)_i E_i(x), returned in
 * the activation dtype) when the sum was accumulated in fp32, e.g. by
 * moe_expert_down_combine.
 *   y32 (device) [n] fp32;  y (device) [n] bf16 out;  both 16-byte aligned.
 *   clear 1: y32[i] is set to 0 once read, so that it can take the next sum with
 *         moe_expert_down_combine(..., accumulate = 1) and no separate clearing pass;
 *         0: y32 is left as it is.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_round_output(float* y32, int64_t n, void* y, int32_t clear, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_combine -- y[t] = sum_j g_j * y_rows[row_of[t, j]]  (+ shared_y[t]).
 * [MoE-Explained] section "什么是稀疏性？", eq. y = sum_i G(x)_i E_i(x).
 *   y_rows    (device) [rows_max, d] rows_dtype
 *   row_of    (device) [T, k]: -1 slots are skipped (a dropped assignment adds 0)
 *   topk_gate (device) [T, k] fp32, or NULL when y_rows already carry their gate
 *   shared_y  (device) [T, d] rows_dtype or NULL: added with weight 1
 *   y         (device) [T, d] y_dtype out
 *   A row index >= rows_max is skipped (adds 0) and recorded as MOE_DEVERR_ROW.
 * ---------------------------------------------------------------------------------- */
MOE_API moe_status moe_combine(const void* y_rows, int32_t rows_dtype, const int32_t* row_of,
                       const float* topk_gate, const void* shared_y, int32_t T, int32_t d,
                       int32_t k, int64_t rows_max, int32_t y_dtype, void* y, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_router_stats -- load-balance and stability statistics of one routing.
 * [MoE-Explained] auxiliary load-balancing loss (sections on token load balancing and
 * "Switch Transformer"), router z-loss (section "使用路由器 Z-loss 稳定训练");
 * [Handbook-Article] monitoring of max/mean load and drop rate.
 *   logits (device) [T, E] fp32; counts, kept (device) [E] int32 (from moe_histogram_scan)
 *   load   (device) [E] fp32 out: f_e = counts[e] / (T k)
 *   stats5 (device) [5] fp32 out: { aux = E sum_e f_e P_e,  z = mean_t lse_t^2,
 *          dropped = T k - sum kept,  max_over_mean = max counts / (T k / E),
 *          cv = std(counts) / mean(counts) }
 *   P_e is the token-mean of softmax(l) (softmax scoring) or of s / sum_e s.
 *   workspace (device) >= moe_router_stats_workspace_bytes(T, E) bytes.
 * ---------------------------------------------------------------------------------- */
MOE_API size_t moe_router_stats_workspace_bytes(int32_t T, int32_t E);
MOE_API moe_status moe_router_stats(const float* logits, const int32_t* counts, const int32_t* kept,
                            int32_t T, int32_t E, int32_t k, int32_t score,
                            float* load, float* stats5,
                            void* workspace, size_t workspace_bytes, void* stream);

/* moe_zero -- clears `bytes` bytes at p (device) with cudaMemsetAsync on stream: the
 * initial value for moe_expert_down_combine(..., accumulate = 1) when the caller wants
 * to clear y off the critical path (e.g. on a second stream).  p must be 16-byte
 * aligned; bytes = 0 does nothing.  This step has no counterpart on the pages (it only
 * initialises an output buffer). */
MOE_API moe_status moe_zero(void* p, size_t bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_quantize_fp4_host / moe_dequantize_fp4_host -- 4-bit expert weights, packed on the
 * host once at load time.
 * [Handbook-Digest] "已确认", bullet "量化与推理" (Kimi K3's routed experts in MXFP4;
 * NVIDIA's NVFP4 training with key layers in BF16).  Formats:
 *   element  FP4 E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), w / scale rounded to
 *            nearest, ties to the even mantissa bit, magnitudes above 6 saturating;
 *   MXFP4    32-element blocks, scale 2^E stored as the byte E + 127 (E8M0),
 *            E = floor(log2 amax_block) - 2 clamped to [-127, 127] (-127 if all zero);
 *   NVFP4    16-element blocks, scale byte = FP8 E4M3 of amax_block / 6 / s_t (nearest
 *            even, saturating at 448), and one fp32 tensor scale s_t = amax / (6 * 448)
 *            (1 if all zero); a block whose scale rounds to 0 stores zeros.
 *   W            (host) [rows, K] fp32, row-major (the K-major weight: W_gu or W_dn rows)
 *   codes        (host) [rows, K/2] bytes: element 2j in the low nibble of byte j
 *   scales       (host) [rows, K/block] bytes, block = moe_fp4_block_size(fmt)
 *   tensor_scale (host) one fp32 (NVFP4 only; may be NULL for MXFP4)
 *   threads      host threads (0 = all cores); the result does not depend on it
 * Both run on the host and return when done (no stream, no launch).  Dequantization
 * returns code value x block scale (x tensor scale), rounded to fp32.
 * Errors: INVALID_ARG for a null pointer, negative sizes or threads, or an unknown format;
 * UNSUPPORTED when K is not a multiple of the block.  No device memory is touched.
 * ---------------------------------------------------------------------------------- */
MOE_API int32_t moe_fp4_block_size(int32_t fmt);
MOE_API moe_status moe_quantize_fp4_host(const float* W, int64_t rows, int64_t K, int32_t fmt,
                     uint8_t* codes, uint8_t* scales, float* tensor_scale, int32_t threads);
MOE_API moe_status moe_dequantize_fp4_host(const uint8_t* codes, const uint8_t* scales,
                     const float* tensor_scale, int64_t rows, int64_t K, int32_t fmt,
                     float* W, int32_t threads);

/* ------------------------------------------------------------------------------------
 * moe_expert_gate_up_fp4 / moe_expert_down_fp4 -- the grouped expert GEMMs with 4-bit
 * expert weights (weight-only: activations, H and the gated rows stay as in the bf16
 * calls).  [Handbook-Digest] "已确认", bullet "量化与推理" (routed experts in MXFP4;
 * NVFP4 with key layers kept in BF16).
 * The weights are the packed form of moe_quantize_fp4_host, in device memory, with the
 * scales rearranged once by moe_prepare_fp4_scales:
 *   codes         (device) [rows, K/2] bytes (element 2j in the low nibble of byte j)
 *   scales        (device) the prepared scales: moe_fp4_scales_bytes(rows, K, fmt) bytes
 *   tensor_scale  (device) [E] fp32, expert e's NVFP4 tensor scale (quantize each expert
 *                 separately); NULL for MXFP4
 *   gate/up: rows = E * 2F (expert e's F gate rows, then its F up rows), K = d;
 *   down:    rows = E * d, K = F.
 * Every weight is code value x block scale (x tensor scale).  The kernel expands each
 * stage of codes to bf16 in shared memory (exact: at most 6 significant bits) and runs
 * the bf16 tensor-core MMAs with fp32 accumulation; the NVFP4 tensor scale multiplies the
 * accumulators.  Weight-major tiles (256 weight rows x the expert's tokens), whatever the
 * group sizes.  Other arguments as moe_expert_gate_up / moe_expert_down (bf16 rows only).
 * Errors: INVALID_ARG for a null pointer, a bad format, a missing NVFP4 tensor scale or a
 * negative size; UNSUPPORTED for E > 1024, d or F not a multiple of 64, fp32 activations
 * or an unaligned pointer.
 * ---------------------------------------------------------------------------------- */
/* moe_prepare_fp4_scales -- the 4-bit GEMMs' scale layout, made once at load time.
 *   scales  (device) [rows, K / block] bytes as moe_quantize_fp4_host writes them
 *   out     (device) moe_fp4_scales_bytes(rows, K, fmt) bytes, 16-byte aligned: k-block
 *           major, out[kb][row][j] = scales[row][kb * (64 / block) + j] for the K/64
 *           k-blocks of 64 elements, followed in each k-block by 256 zero rows, so that one
 *           k-block's scales of 128 consecutive rows are one contiguous copy.
 * moe_fp4_scales_bytes returns 0 for a bad format, negative sizes or K % 64 != 0.
 * Errors: INVALID_ARG for a null pointer, negative sizes or a bad format; UNSUPPORTED for
 * K % 64 != 0 or an unaligned out; WORKSPACE when bytes is below the query. */
MOE_API size_t moe_fp4_scales_bytes(int64_t rows, int32_t K, int32_t fmt);
MOE_API moe_status moe_prepare_fp4_scales(const uint8_t* scales, int64_t rows, int32_t K, int32_t fmt,
                     uint8_t* out, size_t bytes, void* stream);
MOE_API moe_status moe_expert_gate_up_fp4(const void* x_rows, const int32_t* offsets, int32_t E,
                     int32_t d, int32_t F, int64_t rows_max, const uint8_t* codes,
                     const uint8_t* scales, int32_t fmt, const float* tensor_scale, void* h,
                     void* stream);
MOE_API moe_status moe_expert_down_fp4(const void* h, const int32_t* offsets, int32_t E, int32_t d,
                     int32_t F, int64_t rows_max, const uint8_t* codes, const uint8_t* scales,
                     int32_t fmt, const float* tensor_scale, const float* gate_of_row,
                     int32_t y_dtype, void* y_rows, void* stream);

/* Largest workspace any of the calls above needs for these sizes, for every call with
 * at most T tokens (each size query covers the batches below its T). */
MOE_API size_t moe_workspace_bytes(int32_t T, int32_t d, int32_t E, int32_t k);

/* Reads and clears the current device's error word (synchronises `stream`).
 * *code = MOE_DEVERR_*; returns MOE_ERR_DEVICE when *code != 0, else MOE_OK. */
MOE_API moe_status moe_get_device_error(int32_t* code, void* stream);

/* Human-readable names. */
MOE_API const char* moe_status_str(int32_t status);
MOE_API const char* moe_last_cuda_error(void);

/* Library version (major * 10000 + minor * 100 + patch). */
MOE_API int32_t moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
