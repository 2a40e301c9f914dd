/*
 * moe_mx.h -- C ABI of libmoe_mx.so, a fused routed mixture-of-experts layer
 * with OCP MXFP4 expert weights for NVIDIA B200 (sm_100a).
 *
 * One call, moe_mx_forward, runs the whole layer on one GPU, on the caller's
 * stream, as hand-written CUDA kernels:
 *   1. top-k softmax routing (lowest expert index wins ties, weights
 *      renormalised to sum to 1)
 *        -- TokenSpeed-kernel README, "Public API" (moe_route); fusedtok
 *           package description, "Operators" and "API stability";
 *   2. grouping of the (token, slot) pairs by expert into a padded layout
 *        -- TokenSpeed-kernel README, "Public API" (moe_dispatch);
 *           mxfp6-sm120 package description, "Execution model" (indirect
 *           routing on the grouped path);
 *   3. FC1 (gate and up projections, MXFP4 weights) with a fused SwiGLU,
 *      h = silu(gate) * up
 *        -- tokenspeed-situ package description, intro ("FC1 MXFP4 + ...")
 *           and "Supported contract"; b12x package description, "What's in
 *           here" (SwiGLU);
 *   4. FC2 (MXFP4 weights)
 *        -- tokenspeed-situ package description, intro (matching FC2);
 *   5. routing-weighted combine, out[t] = sum_j w[t,j] * y[t,j], j ascending
 *        -- TokenSpeed-kernel README, "Public API" (moe_combine).
 * Activations are bf16 (w4a16) or, with MOE_MX_ACT_MXFP8, quantised on the fly
 * to MXFP8 E4M3 with one E8M0 scale per 32 elements (w4a8); on the w4a8 path
 * FC1's output is quantised to MXFP8 and dequantised to bf16 before FC2
 *        -- tokenspeed-situ package description, "Activation precision
 *           (w4a16 vs w4a8)"; mxfp6-sm120 package description, "Execution
 *           model".
 * MX encodings follow the OCP Microscaling Formats (MX) v1.0 specification.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor argument is a plain device pointer to contiguous row-major
 *   memory owned by the caller, 16-byte aligned; sizes are element counts.
 *   Host pointers are rejected with MOE_MX_ERR_INVALID_ARG.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *   stream).  Entry points only enqueue work on it; none synchronises the host
 *   (except the explicitly synchronous helpers noted below).
 * - Return value: MOE_MX_OK (0) or a negative MOE_MX_ERR_* code; the text of
 *   the last error on the calling host thread is moe_mx_last_error().
 *   Arguments are validated on the host before any launch: a rejected call
 *   enqueues nothing.  No entry point traps or aborts the process.
 * - Layout choices the pages leave open, fixed here:
 *   * packed FP4: element 2i is the low nibble of byte i, element 2i+1 the
 *     high nibble;
 *   * w1's 2I rows per expert are the gate rows [0, I) then the up rows
 *     [I, 2I);
 *   * scales are unswizzled row-major [rows, K/32] E8M0 bytes (2^(byte-127)).
 */
#ifndef MOE_MX_H
#define MOE_MX_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_MX_API __attribute__((visibility("default")))
#else
#define MOE_MX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define MOE_MX_OK 0
#define MOE_MX_ERR_INVALID_ARG (-1) /* null/host/misaligned pointer, bad size or enum */
#define MOE_MX_ERR_UNSUPPORTED (-2) /* device is not sm_100, or a shape outside the supported set */
#define MOE_MX_ERR_CUDA (-3)        /* a CUDA runtime/driver call failed; text in moe_mx_last_error */
#define MOE_MX_ERR_TIMEOUT (-4)     /* a bounded device-side wait gave up (see moe_mx_sync_status) */
#define MOE_MX_ERR_NO_MEMORY (-5)   /* workspace allocation failed in moe_mx_create */

/* Activation precision (act_dtype). */
#define MOE_MX_ACT_BF16 0  /* w4a16: bf16 activations x MXFP4 weights */
#define MOE_MX_ACT_MXFP8 1 /* w4a8: activations quantised to MXFP8 E4M3 before FC1 */

/* Output element type of moe_mx_forward_routed (out_dtype). */
#define MOE_MX_OUT_BF16 0 /* bf16 [T, H] */
#define MOE_MX_OUT_F32 1  /* float32 [T, H]: a shard's partial output, for a sum over shards */

/* Element formats for moe_mx_quantize. */
#define MOE_MX_FMT_MXFP4 0 /* E2M1 codes, two per byte */
#define MOE_MX_FMT_MXFP8 1 /* E4M3 codes, one per byte */

/* Layouts of the E8M0 weight scales moe_mx_forward reads (moe_mx_set_scale_layout). */
#define MOE_MX_SCALES_ROW_MAJOR 0 /* [E, rows, K/32] as the quantiser writes them (default) */
#define MOE_MX_SCALES_TILED 1     /* rearranged by moe_mx_prepare_scales */

/* Which expert weight a scale tensor belongs to (moe_mx_prepare_scales). */
#define MOE_MX_W1 0 /* [E, 2I, H/32]: gate rows then up rows */
#define MOE_MX_W2 1 /* [E, H, I/32] */

typedef struct moe_mx_handle moe_mx_handle;

/*
 * Create a layer handle for fixed dimensions and allocate its workspace on
 * `device` (the workspace is sized once, for max_tokens tokens and
 * max_top_k slots; moe_mx_forward never allocates).
 *   hidden      H, the model dimension: a multiple of 128, 128..16384.
 *   inter       I, the expert intermediate dimension: a multiple of 128,
 *               128..8192.
 *   num_experts E: 1..1024.
 *   max_tokens  largest num_tokens a forward will be given: 1..65536.
 *   max_top_k   largest top_k a forward will be given: 1..32 (moe_mx_forward
 *               also needs top_k <= E; moe_mx_forward_routed does not).
 *   device      CUDA device ordinal; must be compute capability 10.0.
 * On success *out receives the handle (caller owns it; free it with
 * moe_mx_destroy).  Errors: INVALID_ARG, UNSUPPORTED, NO_MEMORY, CUDA.
 */
MOE_MX_API int moe_mx_create(moe_mx_handle **out, int hidden, int inter, int num_experts, int max_tokens,
                  int max_top_k, int device);

/*
 * moe_mx_create with a shared expert (mxfp6-sm120 package description, routed-MoE
 * path: "shared-expert combine and routed/shared reduction"): every token also
 * passes through a shared SwiGLU expert of intermediate size num_shared * inter,
 * whose output is added to the routed sum with weight 1 in the same combine.
 *   num_shared  S >= 0: the shared expert is held as S chunks of `inter` in
 *               expert slots num_experts .. num_experts + S - 1 of the weight
 *               tensors, which then hold num_experts + S slots ([E + S, ...]).
 *               Chunk c holds gate rows c*I .. c*I + I - 1 of the shared W1
 *               followed by the matching up rows, and columns c*I .. c*I + I - 1
 *               of the shared W2 (SwiGLU acts element by element along the
 *               intermediate dimension, so the chunks' outputs add up to the
 *               shared expert's output).  S = 0 is moe_mx_create.
 * The router sees the routed experts only: router_logits stay [T, num_experts].
 * A token has top_k + S slots; moe_mx_get_routing reports them in that order
 * (the shared slots: ids num_experts.., weight 1) and counts / pad_offsets over
 * all E + S slots.  num_experts + S <= 1024 and max_top_k + S <= 32, else
 * MOE_MX_ERR_UNSUPPORTED.  moe_mx_forward_routed takes no shared expert
 * (a handle with S > 0 rejects it with MOE_MX_ERR_UNSUPPORTED).
 */
MOE_MX_API int moe_mx_create_ex(moe_mx_handle **out, int hidden, int inter, int num_experts, int num_shared,
                                int max_tokens, int max_top_k, int device);

/*
 * Run the layer: out = MoE(x) for num_tokens tokens, enqueued on `stream`.
 *   x              bf16 [T, H] activations.
 *   router_logits  float32 [T, E] router logits (any per-expert bias already
 *                  folded in).
 *   num_tokens     T: 0..max_tokens (T = 0 returns MOE_MX_OK and enqueues
 *                  nothing).
 *   w1             MXFP4 codes  [E, 2I, H/2] bytes (gate rows, then up rows).
 *   w1_scale       E8M0 scales  [E, 2I, H/32] bytes.
 *   w2             MXFP4 codes  [E, H, I/2] bytes.
 *   w2_scale       E8M0 scales  [E, H, I/32] bytes.
 *   top_k          k: 1..min(E, max_top_k).
 *   act_dtype      MOE_MX_ACT_BF16 or MOE_MX_ACT_MXFP8.
 *   out            bf16 [T, H], written (not accumulated); must not alias x.
 * Only experts that receive at least one token have their weights read.
 * Weight scale bytes are E8M0 (2^(byte-127)); the tensor core applies them
 * together with the activations' block scales and accumulates in float32.
 * Every byte 0..254 is valid: products below float32's normal range may be
 * flushed to zero and sums beyond its range become infinite; the NaN byte 0xFF
 * makes every output it reaches NaN.  An activation block holding a NaN or an
 * infinity is encoded with the NaN scale byte (see moe_mx_debug_encode_act),
 * so the outputs of that token come out NaN.
 * The call does not synchronise the host, allocates nothing and may be
 * captured in a CUDA graph.  One forward may be in flight per handle.
 * Device-side failures (a bounded wait that gave up) surface through
 * moe_mx_sync_status.  Errors: INVALID_ARG, CUDA.
 */
MOE_MX_API int moe_mx_forward(moe_mx_handle *h, const void *x, const float *router_logits, int num_tokens,
                   const uint8_t *w1, const uint8_t *w1_scale, const uint8_t *w2,
                   const uint8_t *w2_scale, int top_k, int act_dtype, void *out, void *stream);

/*
 * Run the layer with the routing given instead of computed, for one contiguous
 * shard of the experts: precomputed, unpacked top-k (global expert ids and
 * their weights), experts outside the shard filtered out, and the shard's
 * partial output written (tokenspeed-situ package description, "Supported
 * contract": precomputed top-k routing, global expert ids, contiguous local
 * expert shards with a local expert offset, the native routing filtering out
 * other shards' experts into a partial output the caller all-reduces).  The
 * handle's E is the number of local experts; the weights hold those E experts.
 *   x                    bf16 [T, H] activations.
 *   topk_ids             int32 [T, k] global expert ids; an id in
 *                        [local_expert_offset, local_expert_offset + E) selects
 *                        local expert id - local_expert_offset, any other value
 *                        (another shard's expert, or no expert) adds nothing.
 *                        Ids of one token need not be distinct or ordered.
 *   topk_w               float32 [T, k] the routing weights, used as given (no
 *                        renormalisation).
 *   num_tokens           T: 0..max_tokens (0: MOE_MX_OK, nothing enqueued).
 *   top_k                k: 1..max_top_k (may exceed E).
 *   local_expert_offset  >= 0: global id of local expert 0.
 *   w1, w1_scale, w2, w2_scale, act_dtype: as for moe_mx_forward, [E, ...].
 *   out                  [T, H], written (not accumulated), must not alias x:
 *                        bf16 (out_dtype MOE_MX_OUT_BF16) or float32
 *                        (MOE_MX_OUT_F32, the partial sum before rounding, so
 *                        that the partial outputs of all shards add up to the
 *                        layer's output with one rounding at the end).
 *                        out[t] = sum over slots j of token t whose expert is
 *                        local, j ascending, of topk_w[t,j] * FC2(SwiGLU(FC1(x[t]))).
 * moe_mx_get_routing afterwards reports the local ids (-1 for slots outside
 * the shard) and the given weights; counts and the grouping cover the local
 * pairs only.  Allocation, synchronisation, graph capture and errors as for
 * moe_mx_forward (INVALID_ARG also for a bad out_dtype or a negative offset).
 */
MOE_MX_API int moe_mx_forward_routed(moe_mx_handle *h, const void *x, const int32_t *topk_ids, const float *topk_w,
                                     int num_tokens, int top_k, int local_expert_offset, const uint8_t *w1,
                                     const uint8_t *w1_scale, const uint8_t *w2, const uint8_t *w2_scale,
                                     int act_dtype, void *out, int out_dtype, void *stream);

/*
 * Run the layer over one rank's contiguous shard of the experts, routed from the
 * whole layer's router logits: expert parallelism as the tokenspeed-situ package
 * description's "Supported contract" runs it (every rank sees global expert
 * ids, keeps the pairs of its contiguous local shard, and writes a partial
 * output that the caller all-reduces over the expert-parallel group), with the
 * routing done here, on every rank, for all tokens.  The handle's E is the number
 * of local experts; the weights hold those E experts.
 *   router_logits       float32 [T, num_experts_global], the whole layer's logits.
 *   num_experts_global  experts of the whole layer: 1..1024, >= local_expert_offset + E.
 *   local_expert_offset global id of local expert 0 (>= 0).
 *   top_k               1..min(num_experts_global, max_top_k): the whole layer's
 *                       top-k (softmax, lowest index winning ties, weights
 *                       renormalised over the k), as moe_mx_forward chooses it.
 *   out                 [T, H], written: float32 (MOE_MX_OUT_F32: the shard's
 *                       partial sum, sum over slots j whose expert is local of
 *                       w[t,j] * FC2(SwiGLU(FC1(x[t]))), j ascending; the partial
 *                       outputs of all shards add up to the layer's output before
 *                       its rounding) or bf16 (MOE_MX_OUT_BF16).
 *   x, w1, w1_scale, w2, w2_scale, act_dtype, num_tokens: as for moe_mx_forward.
 * With the shard [0, E) of E experts this is moe_mx_forward (same routing, same
 * output bits for bf16).  moe_mx_get_routing afterwards reports the local ids
 * (-1 for a selected expert outside the shard) and the whole layer's weights.
 * Allocation, synchronisation, graph capture and errors as for moe_mx_forward
 * (INVALID_ARG also for a bad out_dtype or a shard outside the layer;
 * UNSUPPORTED for a handle with a shared expert).
 */
MOE_MX_API int moe_mx_forward_shard(moe_mx_handle *h, const void *x, const float *router_logits, int num_tokens,
                                    int num_experts_global, int local_expert_offset, const uint8_t *w1,
                                    const uint8_t *w1_scale, const uint8_t *w2, const uint8_t *w2_scale, int top_k,
                                    int act_dtype, void *out, int out_dtype, void *stream);

/* Free the handle and its workspace (waits for the device).  NULL is a no-op. */
MOE_MX_API int moe_mx_destroy(moe_mx_handle *h);

/* Text of the last error raised on the calling host thread ("" if none). */
MOE_MX_API const char *moe_mx_last_error(void);

/*
 * Synchronise `stream` and read the handle's device error word: MOE_MX_OK,
 * MOE_MX_ERR_TIMEOUT if a kernel's bounded wait gave up since the last call
 * (the word is then cleared), or MOE_MX_ERR_CUDA for an asynchronous CUDA
 * error.  Synchronous.
 */
MOE_MX_API int moe_mx_sync_status(moe_mx_handle *h, void *stream);

/*
 * Quantise a float32 matrix src [rows, K] (K a multiple of 32) to MX along K
 * on the GPU, with the rule the layer's inputs follow: per 32-element block,
 * scale exponent s = floor(log2(amax)) - emax (emax 2 for E2M1, 8 for E4M3),
 * clamped to [-127, 127], E8M0 byte s + 127 (all-zero block: byte 0); codes =
 * round-to-nearest-even of v * 2^-s, saturating at the largest magnitude.
 * (OCP MX v1.0 specification; tokenspeed-situ package description,
 * "Activation precision (w4a16 vs w4a8)".)
 *   fmt MOE_MX_FMT_MXFP4: codes [rows, K/2]; MOE_MX_FMT_MXFP8: codes [rows, K].
 *   scales [rows, K/32].
 * A block holding a NaN or an infinity gets scale byte 0xFF and zero codes.
 * A utility for preparing weights; its MXFP8 path runs the same device encoder
 * as the forward's w4a8 activation quantisation (moe_mx_debug_encode_act, method
 * 0).  Errors: INVALID_ARG, CUDA.
 */
MOE_MX_API int moe_mx_quantize(const float *src, int64_t rows, int64_t K, int fmt, uint8_t *codes,
                    uint8_t *scales, void *stream);

/* ---------------------------------------------------------------------------
 * Inspection entry points (tests and diagnostics).  They copy the routing and
 * grouping state of the most recent forward on `stream` into caller buffers
 * (device pointers); call them after moe_mx_forward on the same stream.
 * ------------------------------------------------------------------------- */

/* Rows of the padded grouped layout per expert segment (128). */
MOE_MX_API int moe_mx_block_rows(void);

/*
 * Number of rows of the padded grouped layout a forward of T tokens and top_k
 * routed slots may occupy at most: P + min(P, E)*(block_rows-1) with P = T*(top_k
 * + S) pairs (S shared chunks, E expert slots), rounded up to block_rows.
 * Host-only arithmetic.
 */
MOE_MX_API int64_t moe_mx_max_grouped_rows(const moe_mx_handle *h, int num_tokens, int top_k);

/*
 * Copy the routing/grouping state of the most recent forward:
 *   topk_ids    int32 [T, k]   selected experts, descending logit;
 *   topk_w      float [T, k]   renormalised weights;
 *   counts      int32 [E]      pairs per expert;
 *   pad_offsets int32 [E+1]    first grouped row of each expert segment;
 *                              segment e spans ceil(counts[e]/128)*128 rows;
 *   sorted_pair int32 [rows]   pair id t*k+j at each grouped row, -1 on
 *                              padding rows; rows = moe_mx_max_grouped_rows
 *                              (entries past pad_offsets[E] are unspecified).
 * Any pointer may be NULL to skip that array.  Errors: INVALID_ARG, CUDA.
 */
MOE_MX_API int moe_mx_get_routing(const moe_mx_handle *h, int32_t *topk_ids, float *topk_w, int32_t *counts,
                       int32_t *pad_offsets, int32_t *sorted_pair, void *stream);

/* Intermediate buffers of a forward (moe_mx_get_intermediate). */
#define MOE_MX_INTER_AQ 0  /* FC1's activation operand: E4M3 codes [2][rows][H] */
#define MOE_MX_INTER_ASF 1 /* its E8M0 scale atoms [rows/128][H/128][2][512] */
#define MOE_MX_INTER_HQ 2  /* FC2's activation operand (h): E4M3 codes [2][rows][I] */
#define MOE_MX_INTER_HSF 3 /* its E8M0 scale atoms [rows/128][I/128][2][512] */
#define MOE_MX_INTER_Y 4   /* FC2's output: float32 [rows][H] */

/*
 * Copy one intermediate buffer of the most recent forward into dst (a device
 * buffer on the handle's device), for tests that check each stage on its own
 * (test-only; the pages print no such interface, the hot-path scope of this
 * library lists it beside moe_mx_get_routing).  rows =
 * moe_mx_max_grouped_rows(h, T, top_k) of that forward; grouped row r holds
 * the pair sorted_pair[r] (moe_mx_get_routing); rows past pad_offsets[E] and
 * padding rows (sorted_pair -1) hold unspecified bytes.
 *   MOE_MX_INTER_AQ / _HQ: the operand as E4M3 codes in two term planes of
 *     rows x K bytes each (K = H for AQ, I for HQ), plane t at t * rows * K.
 *     w4a16 (and h on every path but w4a8): value = term 0 + term 1, an exact
 *     two-term expansion of the bf16 value (see moe_mx_debug_encode_act).
 *     w4a8: term 0 alone is the OCP MXFP8 quantisation; plane 1 is unused.
 *   MOE_MX_INTER_ASF / _HSF: the E8M0 scale bytes of those codes, (rows/128) x
 *     (K/128) atoms of 1024 bytes: for grouped row r, 32-element block b of
 *     the row and term t, the byte at ((r/128) * (K/128) + b/4) * 1024 + t * 512
 *     + (r % 32) * 16 + ((r % 128) / 32) * 4 + b % 4.
 *   MOE_MX_INTER_Y: FC2's float32 output rows before the weighted combine.
 * Asynchronous on `stream`; call it after the forward on the same stream.
 * Errors: INVALID_ARG (bad handle, `which` or dst), CUDA.
 */
MOE_MX_API int moe_mx_get_intermediate(const moe_mx_handle *h, int which, void *dst, void *stream);

/*
 * Run the forward's activation encoders on caller data (test-only; no
 * counterpart on the pages): float32 rows src [rows, K] (K a multiple of 128)
 * become E4M3 codes [2][rows][K] and E8M0 scale atoms [ceil(rows/128)][K/128][2][512]
 * in the layout of MOE_MX_INTER_AQ / _ASF.  Per 32-element block of a row:
 *   act_dtype MOE_MX_ACT_MXFP8: the OCP MXFP8 quantisation (scale exponent
 *     floor(log2 amax) - 8, clamped to [-127, 127]; round-to-nearest-even,
 *     saturating at 448), plane 0 only -- the w4a8 activations and h;
 *   act_dtype MOE_MX_ACT_BF16: each value rounded to bf16, then split exactly
 *     into two MXFP8 terms: term 0 with exponent floor(log2 amax) - 7 keeps the
 *     top 4 significant bits of every element, term 1 the remainder with its own
 *     block exponent (same rule); elements of at least 2^-13 of the block's
 *     maximum are exact, smaller ones err by less than 2^-20 of it -- the w4a16
 *     activations and h;
 *   a block holding a NaN or an infinity: scale byte 0xFF and zero codes in
 *     every term.
 *   method 0: one thread per block, the encoder of the gather (on bf16 values)
 *     and of FC1's epilogue for units with the tokens on the MMA's M side;
 *   method 1: one warp per block, FC1's epilogue for units with the tokens on N.
 * All pointers device memory of the current device, 16-byte aligned.
 * Errors: INVALID_ARG, CUDA.
 */
MOE_MX_API int moe_mx_debug_encode_act(const float *src, int rows, int K, int act_dtype, int method, uint8_t *codes,
                                       uint8_t *scale_atoms, void *stream);

/*
 * Number of kernels the handle's forwards have launched since moe_mx_create
 * (host-side count; -1 for a NULL handle).  The difference across a region is
 * that region's launch count.
 */
MOE_MX_API long long moe_mx_launch_count(const moe_mx_handle *h);

/* Stages of one forward, in launch order (indices into moe_mx_get_stage_times). */
#define MOE_MX_STAGE_ROUTE 0   /* routing, histogram, scan, stable scatter */
#define MOE_MX_STAGE_GATHER 1  /* gather of activation rows (+ MXFP8 quantisation) */
#define MOE_MX_STAGE_FC1 2     /* FC1 grouped GEMM with the SwiGLU epilogue (up to 16 tokens: FC1 and FC2, one launch) */
#define MOE_MX_STAGE_FC2 3     /* FC2 grouped GEMM (empty when it ran in FC1's launch) */
#define MOE_MX_STAGE_COMBINE 4 /* weighted combine */
#define MOE_MX_NUM_STAGES 5

/*
 * Enable (1) or disable (0) per-stage timing.  Enabling (again) resets the
 * record.  While enabled, every forward records CUDA events on its stream
 * between its stages (no host synchronisation; a few microseconds of device
 * overhead per forward); the events of the last 1024 timed forwards are kept.
 * Errors: INVALID_ARG, CUDA.
 */
MOE_MX_API int moe_mx_set_stage_timing(moe_mx_handle *h, int enable);

/*
 * Mean per-stage device time, in milliseconds, over the timed forwards kept
 * (at most the last 1024 since timing was enabled): ms[MOE_MX_NUM_STAGES],
 * indexed by MOE_MX_STAGE_*.  Waits for the last timed forward's final event.
 * Errors: INVALID_ARG (timing not enabled or no timed forward yet), CUDA.
 */
MOE_MX_API int moe_mx_get_stage_times(moe_mx_handle *h, float *ms);

/*
 * Weight preparation.  The pages leave tensor preparation to the adapter that owns
 * the weights (TokenSpeed SiTU package description, "Runtime API"); this library
 * offers one such step for the E8M0 weight scales.  The GEMM reads, per 128-row
 * weight tile and 128-element K stage, the 4 scale bytes of each of the 128 rows;
 * in the row-major layout those are 128 scattered 4-byte pieces, in the tiled
 * layout one contiguous 512-byte block (one copy instead of 128).
 *
 * moe_mx_prepare_scales writes the tiled layout of one scale tensor: src is the
 * row-major tensor (which = MOE_MX_W1: [E, 2I, H/32]; MOE_MX_W2: [E, H, I/32]),
 * dst a caller-owned device buffer of the same size; both device pointers on the
 * handle's device, 16-byte aligned, not overlapping.  Asynchronous on `stream`;
 * the codes (w1, w2) are not touched and stay row-major.  Layout of dst: for
 * expert e, weight tile nt and K stage kk, 512 bytes at ((e * n_tiles + nt) *
 * (K/128) + kk) * 512, byte (m % 32) * 16 + (m / 32) * 4 + b = the scale of tile
 * row m, 32-element block b of the stage; W1 tiles (n_tiles = I/64) hold gate
 * rows 64 nt .. 64 nt + 63 then up rows I + 64 nt .. I + 64 nt + 63, W2 tiles
 * (n_tiles = H/128) rows 128 nt .. 128 nt + 127.  Errors: INVALID_ARG, CUDA.
 *
 * moe_mx_set_scale_layout selects which layout the handle's later forwards read
 * from w1_scale and w2_scale (both tensors in the same layout).  Host-only.
 * Errors: INVALID_ARG.
 */
MOE_MX_API int moe_mx_prepare_scales(const moe_mx_handle *h, int which, const uint8_t *src, uint8_t *dst,
                                     void *stream);
MOE_MX_API int moe_mx_set_scale_layout(moe_mx_handle *h, int layout);

/*
 * Self-test of the device watchdog: launch one kernel that waits on a device
 * flag nothing sets, with a wait limit of timeout_us microseconds.  The wait
 * gives up, the kernel records MOE_MX_ERR_TIMEOUT in the handle's error word
 * and returns; moe_mx_sync_status then reports it.  Nothing faults or traps.
 */
MOE_MX_API int moe_mx_debug_watchdog(moe_mx_handle *h, int timeout_us, void *stream);

/*
 * Routing and grouping without a handle and without allocating: the router
 * (softmax, top-k with the lowest expert index winning ties, renormalised
 * weights) and the stable grouping by expert into 128-row padded segments --
 * the same kernels and results as the first stage of moe_mx_forward.  The
 * pages have no counterpart of this entry point; it exists for callers that
 * cannot allocate device memory at the point of the call and hold no handle
 * (for example an op whose device memory must all come from its framework's
 * own pool, where a cudaMalloc would bypass the pool and can synchronise the
 * device).
 *
 * It allocates nothing (no cudaMalloc / cudaFree, no allocating library call).
 * Its scratch (per-chunk expert histograms, the row-block list) is a static
 * device array of 1 MiB, one per device; nothing in it needs to start at zero.
 * A call needs 4*E*ceil(T/64) bytes of histograms plus 16 bytes per 128-row
 * block of the grouped layout (plus 256-byte alignment): at E = 384, top-8
 * that allows about 41,000 tokens.  Larger shapes are rejected with
 * MOE_MX_ERR_UNSUPPORTED and a message giving the limit.
 *
 * The first call on a device looks up that device's scratch address
 * (cudaGetSymbolAddress), which may load the library's device code there: make
 * that first call outside any stream capture (e.g. at setup).  The address is
 * kept for the life of the process: after a cudaDeviceReset of that device it
 * is stale, so do not call this entry point on a device that has been reset.  All calls on one
 * device share the scratch: calls whose executions overlap (unordered streams,
 * several host threads) race on it and corrupt each other's results; order
 * them (one stream, or events).
 *
 * All pointers are device memory of the current device, 16-byte aligned,
 * owned by the caller, and are only read / written on `stream`:
 *   router_logits float [T, E]    input;
 *   topk_ids      int32 [T, k]    selected experts, descending logit;
 *   topk_w        float [T, k]    renormalised weights;
 *   counts        int32 [E]       pairs per expert;
 *   pad_offsets   int32 [E+1]     first grouped row of each expert segment;
 *   sorted_pair   int32 [rows]    pair id t*k+j at each grouped row, -1 on
 *                                 padding rows; rows = T*k + min(T*k, E)*127
 *                                 rounded up to 128 (capacity), of which the
 *                                 first pad_offsets[E] are written;
 *   pos_of_pair   int32 [T*k]     grouped row of each pair.
 * num_tokens = 0 is a no-op.  Errors: INVALID_ARG (bad sizes, host or
 * misaligned pointers), UNSUPPORTED (num_experts > 1024, scratch too small),
 * CUDA (lookup or launch failure; text in moe_mx_last_error).
 */
MOE_MX_API int moe_mx_route_group_noalloc(const float *router_logits, int num_tokens, int num_experts, int top_k,
                                          int32_t *topk_ids, float *topk_w, int32_t *counts, int32_t *pad_offsets,
                                          int32_t *sorted_pair, int32_t *pos_of_pair, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_MX_H */
