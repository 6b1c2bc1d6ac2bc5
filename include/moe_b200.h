/*
 * moe_b200.h - C ABI of the B200 (sm_100a) expert-parallel MoE layer hot path.
 *
 * The layer, in the order the calls run:
 *
 *   1. moe_route_topk          router top-k with renormalised softmax weights
 *   2. moe_capacity_clip       per-expert token capacity, lowest-weight excess dropped
 *   3. moe_dispatch_layout     expert-contiguous, EP-rank-grouped receive layout,
 *                              the all_to_all_single split counts, optional host copy
 *   4. moe_permute             token rows -> receive rows
 *   5. moe_grouped_swiglu_ffn  per-expert gate/up GEMM, silu(g)*u, down GEMM
 *   6. moe_combine             weighted sum of each token's expert rows
 *
 * plus moe_forward_chunked, which runs 1-2 once and pipelines 3-6 over token
 * chunks on two streams (dispatch of chunk c+1 overlaps the FFN of chunk c),
 * moe_forward_host, the same layer with its activations in host memory, and
 * moe_forward_chunked_save / moe_layer_backward, the forward that keeps the
 * dispatch outputs and the layer's backward that reads them or recomputes them.
 *
 * Also: routing variants through moe_config (grouped top-k, a bias that steers
 * the selection only); moe_shared_expert_ffn, a dense shared expert whose rows
 * the combine adds; moe_dispatch_layout_noalloc, step 3 with its scratch in a
 * fixed library array; moe_quantize_fp8_rows, moe_permute_quantize_fp8 and
 * moe_grouped_swiglu_ffn_fp8, the expert FFN on E4M3 codes with UE8M0 row
 * scales (cfg->ffn_fp8 = 1); moe_quantize_fp8_blocks,
 * moe_permute_quantize_fp8_blocks and moe_grouped_swiglu_ffn_mxfp8, the same
 * with one UE8M0 scale per 32 K values and h quantised inside the SwiGLU
 * epilogue (cfg->ffn_fp8 = 2);
 * moe_grouped_swiglu_ffn_backward, the expert FFN's backward (data and
 * weight gradients); moe_combine_backward, moe_route_backward and
 * moe_permute_backward, the backward's row passes; moe_watchdog_selftest, which makes a bounded wait run
 * out on purpose; moe_device_status, the device-side error bits.
 *
 * Sources (restated, not copied):
 *   [AX]  axolotl docs, "integrations.expert_parallel.args", ExpertParallelArgs:
 *         expert_parallel_backend (torch = all_to_all_single over the EP group),
 *         expert_parallel_dispatch_chunks, expert_parallel_save_dispatch
 *         (the routing choice and the host-side split counts are kept
 *         either way),
 *         expert_parallel_size, expert_parallel_token_capacity, and
 *         validate_expert_parallel_topology.
 *   [LL]  LightLLM PR 1687 review page: _select_experts / norm_topk_prob,
 *         grouped top-k in experts(), the expert prefix-sum ("psum") contiguous
 *         layout of the grouped GEMM, silu_and_mul between the grouped GEMMs,
 *         decode reducing expert outputs straight into a dense output, the
 *         shared expert overlapped with and added in the combine, comm-stream /
 *         compute-stream ownership with record_stream, and dispatch capacity
 *         sized from the padded worst case.
 *
 * Conventions that hold for every call:
 *   - All pointers are DEVICE pointers unless the parameter name ends in
 *     _host.  The caller allocates and owns every buffer, including the
 *     workspace; the library never allocates or frees device memory and never
 *     synchronises the device.  Every call is asynchronous on its stream(s).
 *   - Layouts are row-major and dense.  x, xr, h, y, out, w13 and w2 hold
 *     cfg->dtype elements (MOE_F32: float, MOE_BF16: bfloat16 bit patterns).
 *   - Host-side argument errors return immediately and launch nothing.
 *     Launch failures return MOE_ERR_CUDA.  Conditions only the device can see
 *     (a non-finite logit, a bounded wait that ran out) set bits in the status
 *     word inside the workspace; read them with moe_device_status.  No kernel
 *     traps.
 *   - moe_last_error_detail() describes the last non-OK status of the calling
 *     thread.
 *   - Workspace: a caller-owned device buffer of moe_workspace_bytes(cfg)
 *     bytes (moe_forward_workspace_bytes(cfg) for moe_forward_chunked,
 *     moe_forward_host_workspace_bytes(cfg) for moe_forward_host),
 *     256-byte aligned, zero-filled ONCE before its first use.  A workspace
 *     serves one stream (or one moe_forward_chunked stream pair) at a time.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* bad pointer, size or topology; nothing launched */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but outside the library's limits (below) */
    MOE_ERR_WORKSPACE = 3,    /* workspace pointer misaligned                    */
    MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed            */
    MOE_ERR_DEVICE = 5        /* the device status word has bits set             */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Device status bits (moe_device_status). */
#define MOE_DEV_NONFINITE_LOGIT 0x1u  /* a logit (+bias) was NaN or +-Inf          */
#define MOE_DEV_WAIT_TIMEOUT    0x2u  /* a bounded wait ran out (mbarrier)         */
                                      /* gave up; outputs of that call are invalid */
#define MOE_DEV_BAD_INDEX       0x4u  /* an expert id outside [0, E) was read      */

/*
 * Layer shape.  T tokens, hidden size H, E experts, top-k k, FFN intermediate
 * size I, ep logical EP ranks ([AX] expert_parallel_size; rank d owns the
 * contiguous experts [d*E/ep, (d+1)*E/ep)), capacity per expert per forward
 * ([AX] expert_parallel_token_capacity; < 0 = no cap), n_chunks dispatch
 * chunks ([AX] expert_parallel_dispatch_chunks), reduce_dense = 1 for the
 * decode form in which the FFN reduces w*y straight into a dense fp32 [T, H]
 * buffer ([LL] decode reduce) instead of storing y.
 *
 * Topology checks ([AX] validate_expert_parallel_topology, restated):
 * T >= 0, H, E, k, I, ep, n_chunks >= 1, k <= E, E % ep == 0,
 * T % n_chunks == 0, (T / n_chunks) % ep == 0 (each chunk splits into equal
 * contiguous source-rank blocks).
 * Routing-variant checks (MOE_ERR_INVALID_ARG): n_group >= 0, E % n_group == 0,
 * topk_group and k as stated at the fields, group_score in {0, 1},
 * bias_select_only in {0, 1}, shared_I >= 0 (a multiple of 64 for MOE_BF16, of
 * 4 for MOE_F32).
 * Limits (MOE_ERR_UNSUPPORTED): k <= 32, E <= 1024, ep <= E, T*k < 2^30,
 * n_group <= 32; ffn_fp8 = 1 or 2 only with MOE_BF16, H % 128 == I % 128 == 0
 * and shared_I = 0 (2: also E <= 512 and H <= 8192);
 * MOE_BF16 needs H % 64 == 0 and I % 64 == 0 (tensor-core tiles);
 * MOE_F32 needs H % 4 == 0 and I % 4 == 0.
 */
typedef struct {
    int32_t T, H, E, k, I, ep;
    int32_t capacity;
    int32_t dtype;          /* moe_dtype */
    int32_t n_chunks;
    int32_t reduce_dense;
    /* Routing variants (LightLLM PR 1687: the experts() path keeps "grouped
     * top-k" for DeepSeek-V2, GLM-4-MoE-Lite and Qwen3-MoE).  All zero gives
     * plain top-k with the bias in both selection and weights.
     *   n_group      experts form n_group contiguous groups of E / n_group
     *                (<= 1: no grouping); a token first keeps the topk_group
     *                groups with the best group score, then takes its top-k
     *                among their experts.
     *   topk_group   groups kept per token (1 <= topk_group <= n_group,
     *                k <= topk_group * E / n_group).
     *   group_score  0: a group's score is its best biased logit; 1: the sum of
     *                its two best (E / n_group >= 2).  Groups rank by score,
     *                lower group index first among equal scores.
     *   bias_select_only  1: the bias steers the selection (experts and groups)
     *                only; the weights are the softmax of the unbiased logits of
     *                the chosen experts. */
    int32_t n_group;
    int32_t topk_group;
    int32_t group_score;
    int32_t bias_select_only;
    /* Shared expert ([LL]: shared expert overlap kept in the combine): its
     * intermediate size (0: none).  One dense SwiGLU expert with weights
     * w13_shared [2*shared_I, H] and w2_shared [H, shared_I] applied to every
     * token; its output is added into the combine's sum. */
    int32_t shared_I;
    /* FP8 expert FFN ([LL]: the FP8 grouped GEMM with UE8M0 scales over the
     * psum layout, silu_and_mul followed by quantisation): 1 runs step 5 on
     * E4M3 codes with one UE8M0 (power-of-two) scale per row, see
     * moe_quantize_fp8_rows; the permuted rows are then E4M3 codes.  2 runs
     * it with one UE8M0 scale per row and 32 K values (moe_quantize_fp8_blocks,
     * moe_grouped_swiglu_ffn_mxfp8).  Needs dtype MOE_BF16, H and I multiples
     * of 128 and shared_I = 0. */
    int32_t ffn_fp8;
} moe_config;

/* Validates cfg (topology and limits).  MOE_OK or the reason it is rejected. */
moe_status moe_config_check(const moe_config *cfg);

/* Scratch bytes the step calls need (status word, scan state, thresholds,
 * tile scheduler).  0 if cfg is invalid. */
size_t moe_workspace_bytes(const moe_config *cfg);

/* Bytes moe_forward_chunked needs: the scratch above plus two chunk slots of
 * layout arrays, xr, h and y, and the dense fp32 reduce buffer in decode form
 * (with ffn_fp8: also x's codes and scales, h's codes and scales).  0 if cfg
 * is invalid. */
size_t moe_forward_workspace_bytes(const moe_config *cfg);

/* Worst-case receive rows of one call over tok_count tokens:
 * min(tok_count * k, E * capacity) (capacity >= 0), else tok_count * k.
 * Receive buffers (recv_token, recv_slot, xr, h, y) need this many rows; it is
 * the padded worst case, not the count of the current batch ([LL] decode
 * dispatch capacity).  -1 if cfg is invalid. */
int64_t moe_max_recv_rows(const moe_config *cfg, int32_t tok_count);

/*
 * Step 1 - router top-k ([LL] _select_experts with norm_topk_prob; [AX] the
 * routing top-k is saved state, so it is a caller-owned output).
 *   logits   fp32 [T, E]; bias fp32 [E] or NULL (added to the logits before
 *            selection and weighting).
 *   topk_idx int32 [T, k]: experts by (logit+bias) descending, the lower expert
 *            index first among equal values; slot j = rank j.
 *   topk_w   fp32 [T, k]: w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0), i.e.
 *            the softmax restricted to the top k and renormalised.  The
 *            exponential is a fixed Cody-Waite + degree-7 Taylor evaluation in
 *            fp32 and the sum runs in slot order, so the weights are
 *            bit-reproducible.
 *   counts   int32 [E]: assignments per expert (before the clip).
 * A non-finite logit sets MOE_DEV_NONFINITE_LOGIT; that token's outputs are
 * then unspecified.
 */
moe_status moe_route_topk(const moe_config *cfg, const float *logits, const float *bias,
                          int32_t *topk_idx, float *topk_w, int32_t *counts,
                          void *ws, cudaStream_t stream);

/*
 * Step 2 - per-expert capacity ([AX] expert_parallel_token_capacity): an
 * expert that received more than C = cfg->capacity assignments keeps the C
 * with the largest topk_w and drops the rest; among equal weights the higher
 * token index is dropped first.  Kept weights are not renormalised.
 *   topk_idx, topk_w, counts: outputs of step 1 over all T tokens.
 *   keep        uint8 [T, k]: 1 kept, 0 dropped.
 *   kept_counts int32 [E].
 * With capacity < 0 every assignment is kept.  The clip always runs over the
 * whole forward (all T tokens), before any chunking.
 */
moe_status moe_capacity_clip(const moe_config *cfg, const int32_t *topk_idx,
                             const float *topk_w, const int32_t *counts, uint8_t *keep,
                             int32_t *kept_counts, void *ws, cudaStream_t stream);

/*
 * Step 3 - dispatch layout of the tokens [tok_begin, tok_begin + tok_count)
 * ([AX] torch backend: all_to_all_single over the EP group; [LL] psum layout).
 * The ep ranks are logical: source rank s holds the chunk's tokens
 * [tok_begin + s*tok_count/ep, tok_begin + (s+1)*tok_count/ep) and destination
 * rank d owns experts [d*E/ep, (d+1)*E/ep).  Receive rows are ordered by
 * (destination rank, expert, token), which is the all_to_all_single arrival
 * order regrouped by expert, and equals the stable order by (expert, token).
 *   expert_offsets int32 [E+1]: rows of expert e are [expert_offsets[e],
 *                  expert_offsets[e+1]); expert_offsets[E] = N.
 *   rank_offsets   int32 [ep+1]: rank_offsets[d] = expert_offsets[d*E/ep].
 *   recv_token     int32 [N_max]: absolute token index of each row.
 *   recv_slot      int32 [N_max]: top-k slot of each row.
 *   pos            int32 [tok_count, k]: row of (tok_begin+i, j), -1 if dropped.
 *   send_splits    int32 [ep, ep]: rows source s sends to destination d
 *                  (the receive splits are its transpose).
 *   splits_host    pinned host int32 [E+1 + ep*ep] or NULL: receives
 *                  expert_offsets then send_splits by an async copy on
 *                  `stream` ([AX]: the host-side split counts); valid once
 *                  the stream (or an event recorded after this call) completes.
 * N_max = moe_max_recv_rows(cfg, tok_count).
 */
moe_status moe_dispatch_layout(const moe_config *cfg, int32_t tok_begin, int32_t tok_count,
                               const int32_t *topk_idx, const uint8_t *keep,
                               int32_t *expert_offsets, int32_t *rank_offsets,
                               int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                               int32_t *send_splits, int32_t *splits_host,
                               void *ws, cudaStream_t stream);

/*
 * Allocation-free form of moe_dispatch_layout, for callers that cannot call
 * cudaMalloc or pass a workspace: code running while another framework
 * captures the stream into a CUDA graph, code whose device memory belongs to
 * an allocator it cannot grow, and latency-critical loops that must avoid the
 * implicit synchronisation of cudaMalloc / cudaFree.  The pages describe no
 * such variant; this entry point has no counterpart on them.
 *   Arguments and outputs are those of moe_dispatch_layout, without ws.
 *   status: device uint32 that receives the MOE_DEV_* bits (OR-ed in), or
 *           NULL to drop them.
 * The layout's scratch lives in one fixed device array inside the library
 * (about 256 KiB per device, held until the process exits).  Limits:
 * tok_count <= 16384 (MOE_ERR_UNSUPPORTED beyond).  All calls share the
 * array: calls that may overlap on the GPU race and must be ordered.  The
 * first call on a device looks up the array's address with that device
 * current; make it before any stream capture.  Allocates nothing.
 */
moe_status moe_dispatch_layout_noalloc(const moe_config *cfg, int32_t tok_begin, int32_t tok_count,
                                       const int32_t *topk_idx, const uint8_t *keep,
                                       int32_t *expert_offsets, int32_t *rank_offsets,
                                       int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                                       int32_t *send_splits, int32_t *splits_host,
                                       uint32_t *status, cudaStream_t stream);

/*
 * Step 4 - permute: xr[pos[i, j], :] = x[tok_begin + i, :] for every kept
 * (i, j).  x is [T, H]; xr is [N_max, H]; rows >= N are left untouched.
 * Elements are cfg->dtype, or E4M3 codes (one byte) when cfg->ffn_fp8 = 1.
 */
moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *pos,
                       int32_t tok_begin, int32_t tok_count, void *xr, cudaStream_t stream);

/*
 * Step 5 - grouped SwiGLU FFN over the expert-contiguous rows ([LL] grouped
 * GEMM on the psum layout, silu_and_mul, grouped GEMM).  For each expert e and
 * row p in [expert_offsets[e], expert_offsets[e+1]):
 *   g = W13[e, 0:I, :] . xr[p],  u = W13[e, I:2I, :] . xr[p],
 *   h[p] = silu(g) * u           (stored in cfg->dtype),
 *   y[p] = W2[e] . h[p]          (stored in cfg->dtype).
 *   w13 [E, 2I, H] and w2 [E, H, I]: row-major, K contiguous, used as given.
 *   n_rows: allocated rows of xr, h and y (>= N; normally N_max).
 *   xr [n_rows, H], h [n_rows, I], y [n_rows, H] (y may be NULL in decode form).
 * Decode form (cfg->reduce_dense = 1): y is not stored; instead
 *   out_reduce[recv_token[p], :] += topk_w[recv_token[p], recv_slot[p]] * y[p]
 * in fp32 (out_reduce: fp32 [T, H], zero-filled by the caller; the order of
 * the additions is unspecified).  recv_token, recv_slot and topk_w are only
 * read in decode form.
 * MOE_BF16 runs on tcgen05 tensor cores (bf16 x bf16 -> fp32 in TMEM);
 * MOE_F32 runs fp32 FMA on the CUDA cores.
 */
moe_status moe_grouped_swiglu_ffn(const moe_config *cfg, int64_t n_rows, const void *xr,
                                  const int32_t *expert_offsets, const void *w13,
                                  const void *w2, void *h, void *y,
                                  const int32_t *recv_token, const int32_t *recv_slot,
                                  const float *topk_w, float *out_reduce,
                                  void *ws, cudaStream_t stream);

/*
 * FP8 quantisation by rows ([LL] UE8M0 FP8 quantisation; the E4M3 format has
 * 1 sign, 4 exponent bits with bias 7 and 3 fraction bits, no infinities,
 * largest finite 448).  For each row r of in [rows, cols] (in_dtype MOE_BF16
 * or MOE_F32):
 *   e = the smallest integer with max_c |in[r, c]| <= 448 * 2^e, clamped to
 *       [-126, 127] (0 for a zero row);  scales[r] = e + 127 (UE8M0 byte);
 *   codes[r, c] = E4M3(in[r, c] / 2^e), round to nearest even, magnitudes
 *       beyond 448 saturate to 448.
 * Reading: the pages fix power-of-two scales but not their granularity; one
 * scale per row is taken (per token for activations, per output channel for
 * weights).  A value is codes -> E4M3 value times 2^(scales - 127).  Read as
 * int32, four consecutive scale bytes are the packed form (row 4i in the low
 * byte).  Use it once on W13 ([E*2I, H] rows) and W2 ([E*H, I] rows) for the
 * FP8 FFN, and per call on x.  cols % 8 == 0 (bf16) or % 4 == 0 (fp32).
 * Inputs are expected finite; an infinite row takes e = 127 and saturates.
 */
moe_status moe_quantize_fp8_rows(int64_t rows, int32_t cols, int32_t in_dtype, const void *in,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t stream);

/*
 * Steps 4 and the quantisation of x fused (cfg->ffn_fp8 = 1, cfg->H <= 8192): for
 * t in [tok_begin, tok_begin + tok_count) with at least one kept slot, the bf16
 * row x[t] is quantised as moe_quantize_fp8_rows does (x_scale[t] = its UE8M0
 * byte) and its E4M3 codes are written to every receive row pos[t - tok_begin,
 * j] >= 0 of xr_q [N_max, H].  Rows and scales of tokens without a kept slot are
 * left untouched (x[t] is not read).  The codes and scales equal those of
 * moe_quantize_fp8_rows followed by moe_permute; moe_forward_chunked and
 * moe_forward_host use this form.  MOE_ERR_UNSUPPORTED for H > 8192.
 */
moe_status moe_permute_quantize_fp8(const moe_config *cfg, const void *x, const int32_t *pos,
                                    int32_t tok_begin, int32_t tok_count, uint8_t *xr_q,
                                    uint8_t *x_scale, cudaStream_t stream);

/*
 * Step 5 in FP8 (cfg->ffn_fp8 = 1): the SwiGLU FFN of moe_grouped_swiglu_ffn
 * on E4M3 operands with UE8M0 row scales (value = code * 2^(scale - 127)):
 *   xr_q [n_rows, H]: codes of the receive rows (moe_permute of the codes of
 *        x); x_scale [T]: the scale bytes of x's token rows, read through
 *        recv_token[p];
 *   w13_q [E, 2I, H] with w13_scale [E*2I] (one per weight row), w2_q
 *        [E, H, I] with w2_scale [E*H];
 *   g, u = the dequantised dot products (tcgen05 kind::f8f6f4, fp32 in TMEM,
 *        row and token scales applied to the accumulators);
 *   h [n_rows, I] bf16 = silu(g) * u;  then h_q [n_rows, I], h_scale [n_rows]
 *        = moe_quantize_fp8_rows of h's first N rows (N = expert_offsets[E]);
 *   y [n_rows, H] bf16 = the dequantised W2[e] . h_q[p], or in decode form the
 *        fp32 reduce into out_reduce as in moe_grouped_swiglu_ffn.
 * recv_token is always read; recv_slot and topk_w in decode form only.
 * ws: moe_workspace_bytes(cfg).
 */
moe_status moe_grouped_swiglu_ffn_fp8(const moe_config *cfg, int64_t n_rows, const uint8_t *xr_q,
                                      const uint8_t *x_scale, const int32_t *expert_offsets,
                                      const uint8_t *w13_q, const uint8_t *w13_scale,
                                      const uint8_t *w2_q, const uint8_t *w2_scale, void *h,
                                      uint8_t *h_q, uint8_t *h_scale, void *y,
                                      const int32_t *recv_token, const int32_t *recv_slot,
                                      const float *topk_w, float *out_reduce, void *ws,
                                      cudaStream_t stream);

/*
 * FP8 quantisation with K-blocked scales (LightLLM PR 1687: UE8M0 scales along
 * K, packed four to an int32; the pages give no block length).  Reading: one
 * UE8M0 scale per row and per 32 consecutive values - the block the
 * block-scaled tcgen05 MMA (kind::mxf8f6f4) applies - chosen and applied as
 * moe_quantize_fp8_rows does for a whole row:
 *   scales[r, b] = e + 127 with e the smallest integer such that the largest
 *       |in[r, 32b .. 32b+31]| <= 448 * 2^e (clamped to [-126, 127], 0 for a
 *       zero block);  codes[r, c] = E4M3(in[r, c] / 2^e), nearest even,
 *       saturating.
 *   in [rows, cols] (MOE_BF16 or MOE_F32), cols % 32 == 0; codes [rows, cols];
 *   scales [rows, cols / 32] bytes - four consecutive ones read as an int32
 *   (block 4i in the low byte) are the packed form.
 * Use it once on W13 ([E*2I, H] rows) and W2 ([E*H, I] rows) for
 * moe_grouped_swiglu_ffn_mxfp8.
 */
moe_status moe_quantize_fp8_blocks(int64_t rows, int32_t cols, int32_t in_dtype, const void *in,
                                   uint8_t *codes, uint8_t *scales, cudaStream_t stream);

/*
 * Steps 4 and the K-blocked quantisation of x fused (cfg->ffn_fp8 = 2): for t in
 * [tok_begin, tok_begin + tok_count) with a kept slot, x[t] (bf16) is quantised
 * as moe_quantize_fp8_blocks does and each kept receive row p gets its codes in
 * xr_q [N_max, H] and its block scales in xr_sf [N_max, H/32] (the scales are
 * stored per receive row, beside the codes).  Rows of tokens without a kept slot
 * are left untouched.  Needs H <= 8192.
 */
moe_status moe_permute_quantize_fp8_blocks(const moe_config *cfg, const void *x, const int32_t *pos,
                                           int32_t tok_begin, int32_t tok_count, uint8_t *xr_q,
                                           uint8_t *xr_sf, cudaStream_t stream);

/*
 * Step 5 in FP8 with K-blocked UE8M0 scales (cfg->ffn_fp8 = 2; [LL] the FP8
 * grouped GEMM over the psum layout with UE8M0 scales, and silu_and_mul with the
 * quantisation of its output): value = E4M3(code) * 2^(scale - 127), one scale
 * per row and 32 K values, on every operand:
 *   xr_q [n_rows, H], xr_sf [n_rows, H/32]: the receive rows
 *        (moe_permute_quantize_fp8_blocks);
 *   w13_q [E, 2I, H] with w13_sf [E*2I, H/32], w2_q [E, H, I] with
 *        w2_sf [E*H, I/32] (moe_quantize_fp8_blocks);
 *   g, u = the dequantised dot products (tcgen05 kind::mxf8f6f4 with the block
 *        scales read from TMEM, fp32 accumulation);
 *   h = silu(g) * u rounded to bf16 and quantised by 32-value blocks inside the
 *        same kernel: h_q [n_rows, I] codes, h_sf [n_rows, I/32] (no bf16 h);
 *   y [n_rows, H] bf16 = the dequantised W2[e] . h, or in decode form the fp32
 *        reduce into out_reduce as in moe_grouped_swiglu_ffn.
 * Scale arrays 4-byte aligned.  recv_token, recv_slot, topk_w: decode form only.
 * ws: moe_workspace_bytes(cfg).
 */
moe_status moe_grouped_swiglu_ffn_mxfp8(const moe_config *cfg, int64_t n_rows, const uint8_t *xr_q,
                                        const uint8_t *xr_sf, const int32_t *expert_offsets,
                                        const uint8_t *w13_q, const uint8_t *w13_sf, const uint8_t *w2_q,
                                        const uint8_t *w2_sf, uint8_t *h_q, uint8_t *h_sf, void *y,
                                        const int32_t *recv_token, const int32_t *recv_slot,
                                        const float *topk_w, float *out_reduce, void *ws,
                                        cudaStream_t stream);

/*
 * Step 6 - combine back to token order ([AX] combine all-to-all then the
 * weighted sum): for t in [tok_begin, tok_begin + tok_count)
 *   out[t, :] = sum over j = 0..k-1 with pos[t - tok_begin, j] >= 0 of
 *               topk_w[t, j] * y[pos[t - tok_begin, j], :]
 * accumulated in fp32 in slot order and rounded once to cfg->dtype; a token
 * whose every slot was dropped gets zeros.
 */
moe_status moe_combine(const moe_config *cfg, const void *y, const int32_t *pos,
                       const float *topk_w, int32_t tok_begin, int32_t tok_count,
                       const void *y_shared, void *out, cudaStream_t stream);

/* Decode form of step 6: out[t, :] = round(out_reduce[t, :]) for the tokens
 * [tok_begin, tok_begin + tok_count).
 * In both, y_shared is NULL or the chunk's [tok_count, H] rows of the shared
 * expert's output (moe_shared_expert_ffn, cfg->dtype), added into the fp32 sum
 * before its one rounding. */
moe_status moe_reduce_finalize(const moe_config *cfg, const float *out_reduce,
                               int32_t tok_begin, int32_t tok_count, const void *y_shared,
                               void *out, cudaStream_t stream);

/*
 * The shared expert ([LL]: DeepSeek-style shared expert, its work overlapped
 * with the routed path and its output added in the combine): for the rows
 * t in [tok_begin, tok_begin + tok_count) of x [T, H]
 *   h_shared[t - tok_begin] = silu(Wg x_t) * (Wu x_t)    [tok_count, shared_I]
 *   y_shared[t - tok_begin] = W2s h_shared[t - tok_begin] [tok_count, H]
 * with w13_shared [2*shared_I, H] (gate rows then up rows) and w2_shared
 * [H, shared_I], both cfg->dtype, row-major.  The same kernel as step 5, run
 * as one expert over the chunk's rows (no permutation).  Needs shared_I > 0;
 * ws: moe_workspace_bytes(cfg) (its work counters are not those of step 5, so
 * the two may run on different streams at once).
 */
moe_status moe_shared_expert_ffn(const moe_config *cfg, int32_t tok_begin, int32_t tok_count,
                                 const void *x, const void *w13_shared, const void *w2_shared,
                                 void *h_shared, void *y_shared, void *ws, cudaStream_t stream);

/*
 * Backward steps that are row passes (axolotl ExpertParallelArgs,
 * expert_parallel_save_dispatch: the layer's backward reuses the saved routing
 * top-k, keep mask and layout).  For L = <dout, out>:
 *
 * moe_combine_backward, for t in [tok_begin, tok_begin + tok_count):
 *   dy[pos[t - tok_begin, j]] = topk_w[t, j] * dout[t]     (cfg->dtype, rounded once)
 *   dw[t, j] = <dout[t], y[pos[t - tok_begin, j]]>         (fp32; 0 for a dropped slot)
 *   dout [T, H] and y, dy [N_max, H] in cfg->dtype; dw [T, k]; receive rows no slot
 *   points to are left untouched.  Not for the decode form (y is not stored).
 *
 * moe_route_backward, for every token (the softmax over the k selected logits):
 *   dlogits[t, :] = 0 except dlogits[t, topk_idx[t, j]] = topk_w[t, j] *
 *                   (dw[t, j] - sum_i topk_w[t, i] dw[t, i])     (fp32 [T, E])
 *   dbias (optional, fp32 [E]) = sum over t of dlogits[t, :] in a fixed order,
 *                   or 0 when cfg->bias_select_only.
 *   ws: moe_workspace_bytes(cfg) (an expert id outside [0, E) sets
 *   MOE_DEV_BAD_INDEX and is not written).
 *
 * moe_permute_backward, for t in [tok_begin, tok_begin + tok_count):
 *   dx[t] = sum over kept slots j of dxr[pos[t - tok_begin, j]], fp32 in slot
 *   order, rounded once to cfg->dtype (zeros for a token with every slot
 *   dropped); dxr [N_max, H], dx [T, H].
 */
/*
 * Backward of step 5, the grouped SwiGLU FFN, over one receive buffer (axolotl
 * ExpertParallelArgs, expert_parallel_save_dispatch: the backward of the
 * expert GEMMs under activation checkpointing; the pages give no formulas, the
 * gradient below is that of step 5's function).  For each expert e and row p
 * in [expert_offsets[e], expert_offsets[e+1]) with incoming gradient dy[p]:
 *   g, u   = W13[e, 0:I] . xr[p], W13[e, I:2I] . xr[p]   (recomputed)
 *   dh     = W2[e]^T . dy[p]
 *   h[p]   = silu(g) * u,  s = sigmoid(g)
 *   dg     = dh * u * s * (1 + g * (1 - s)),   du = dh * silu(g)
 *   dxr[p] = W13[e]^T . [dg | du]
 *   dW2[e]  (+)= sum over the expert's rows of dy[p] (x) h[p]       [H, I]
 *   dW13[e] (+)= sum over the expert's rows of [dg | du][p] (x) xr[p] [2I, H]
 *   xr, dy, dxr [n_rows, H]; h [n_rows, I] and dgu [n_rows, 2I] (dg then du)
 *   are outputs kept for the caller; gu [n_rows, 2I] is scratch (g then u; bf16
 *   only, may be NULL for MOE_F32); all in cfg->dtype.
 *   dw13 [E, 2I, H] and dw2 [E, H, I]: fp32, written (accumulate = 0: experts
 *   without rows get zeros) or added to (accumulate = 1).
 * MOE_BF16 runs five tcgen05 launches (g | u; dh with the SwiGLU backward;
 * dxr; the two weight gradients, fp32 accumulation in TMEM, h, dg and du
 * rounded to bf16 where stored); MOE_F32 runs fp32 FMA on the CUDA cores.
 * cfg->ffn_fp8 = 1 is MOE_ERR_UNSUPPORTED.  ws: moe_workspace_bytes(cfg).
 */
moe_status moe_grouped_swiglu_ffn_backward(const moe_config *cfg, int64_t n_rows, const void *xr,
                                           const void *dy, const int32_t *expert_offsets,
                                           const void *w13, const void *w2, void *gu, void *h,
                                           void *dgu, void *dxr, float *dw13, float *dw2,
                                           int32_t accumulate, void *ws, cudaStream_t stream);

moe_status moe_combine_backward(const moe_config *cfg, const void *dout, const void *y,
                                const int32_t *pos, const float *topk_w, int32_t tok_begin,
                                int32_t tok_count, void *dy, float *dw, cudaStream_t stream);
moe_status moe_route_backward(const moe_config *cfg, const int32_t *topk_idx, const float *topk_w,
                              const float *dw, float *dlogits, float *dbias, void *ws,
                              cudaStream_t stream);
moe_status moe_permute_backward(const moe_config *cfg, const void *dxr, const int32_t *pos,
                                int32_t tok_begin, int32_t tok_count, void *dx, cudaStream_t stream);

/*
 * The whole layer, chunked ([AX] expert_parallel_dispatch_chunks; [LL]
 * chunked prefill with comm / compute streams).  Steps 1-2 run once over all
 * T tokens on s_dispatch (the capacity is per forward).  Then for each
 * contiguous chunk c of T/n_chunks tokens, steps 3-4 run on s_dispatch and
 * steps 5-6 on s_compute, so chunk c+1's dispatch overlaps chunk c's FFN.
 * Intermediates live in two chunk slots of the workspace; slot c%2 is reused
 * only after chunk c-2's combine finished.  n_chunks = 1 gives the unchunked
 * layer.  The result equals the unchunked one bit for bit.
 *   logits, bias, x, w13, w2 as in steps 1-5; out [T, H] cfg->dtype.
 *   w13_shared, w2_shared: the shared expert's weights when cfg->shared_I > 0
 *            (else ignored, may be NULL).  Chunk c's shared expert runs on
 *            s_dispatch after its dispatch, beside chunk c's routed FFN on
 *            s_compute, and its rows are added in chunk c's combine.
 *   w13_scale, w2_scale: with cfg->ffn_fp8 = 1, w13 and w2 are E4M3 codes and
 *            these their row scales (moe_grouped_swiglu_ffn_fp8); x stays
 *            bf16 and each chunk's kept rows are quantised inside the permute
 *            (moe_permute_quantize_fp8; for H > 8192 by moe_quantize_fp8_rows
 *            then moe_permute).  With cfg->ffn_fp8 = 2, the block scales of
 *            moe_quantize_fp8_blocks (moe_permute_quantize_fp8_blocks,
 *            moe_grouped_swiglu_ffn_mxfp8).  Else ignored, may be NULL.
 *   topk_idx [T,k], topk_w [T,k], keep [T,k]: caller-owned saved state
 *            ([AX] the routing top-k is always saved).
 *   splits_host: pinned host int32 [n_chunks * (E+1 + ep*ep)] or NULL; chunk c
 *            writes expert_offsets then send_splits at offset c*(E+1+ep*ep).
 *   ws: moe_forward_workspace_bytes(cfg) bytes.
 *   s_dispatch, s_compute: may be the same stream.  On return both streams
 *            are ordered after all the layer's work ([LL] record_stream: the
 *            caller's buffers are touched by both streams, so a caching
 *            allocator must see them used on both).
 */
moe_status moe_forward_chunked(const moe_config *cfg, const float *logits, const float *bias,
                               const void *x, const void *w13, const void *w2,
                               const void *w13_shared, const void *w2_shared,
                               const uint8_t *w13_scale, const uint8_t *w2_scale, void *out,
                               int32_t *topk_idx, float *topk_w, uint8_t *keep,
                               int32_t *splits_host, void *ws,
                               cudaStream_t s_dispatch, cudaStream_t s_compute);

/*
 * moe_forward_chunked that also keeps the dispatch outputs ([AX]
 * expert_parallel_save_dispatch: under activation checkpointing, hold the
 * dispatch / combine all-to-all outputs for the backward instead of issuing
 * the exchanges again): chunk c's receive rows and expert outputs are written
 * to xr_save + c * N_max * H and y_save + c * N_max * H (both [n_chunks,
 * N_max, H] in cfg->dtype, N_max = moe_max_recv_rows(cfg, T / n_chunks); rows
 * past the chunk's N are left untouched).  Otherwise as moe_forward_chunked
 * (same output bits).  Needs ffn_fp8 = 0 and reduce_dense = 0
 * (MOE_ERR_UNSUPPORTED).  ws: moe_forward_workspace_bytes(cfg).
 */
moe_status moe_forward_chunked_save(const moe_config *cfg, const float *logits, const float *bias,
                                    const void *x, const void *w13, const void *w2,
                                    const void *w13_shared, const void *w2_shared, void *out,
                                    int32_t *topk_idx, float *topk_w, uint8_t *keep,
                                    int32_t *splits_host, void *xr_save, void *y_save, void *ws,
                                    cudaStream_t s_dispatch, cudaStream_t s_compute);

/*
 * The layer's backward for L = <dout, out> ([AX] expert_parallel_save_dispatch:
 * the routing top-k and the split counts are always kept; the dispatch and
 * combine outputs are either kept by the forward or produced again).  Chunk by
 * chunk (cfg->n_chunks contiguous token chunks, as the forward ran), on one
 * stream:
 *   1. the chunk's dispatch layout from the saved topk_idx and keep;
 *   2. save mode (xr_saved and y_saved from moe_forward_chunked_save): the
 *      chunk's receive rows and expert outputs are read from them; recompute
 *      mode (both NULL): the rows are permuted again from x and the expert
 *      FFN's forward runs again (the same bits as the forward's);
 *   3. moe_combine_backward (dy rows, the slot gradients dw);
 *   4. moe_grouped_swiglu_ffn_backward (dxr, dW13, dW2);
 *   5. with a shared expert, its backward over the chunk's rows of x with
 *      dy = dout (dW13_shared, dW2_shared, its dx rows);
 *   6. dx[t] = the sum of the token's kept receive-row gradients plus its
 *      shared-expert row (fp32, one rounding to cfg->dtype);
 * then moe_route_backward over all T (dlogits fp32 [T, E]; dbias fp32 [E] or
 * NULL, 0 when cfg->bias_select_only).  The weight gradients (fp32, the
 * layouts of w13 / w2 / w13_shared / w2_shared) are written by the first chunk
 * (added to when accumulate = 1) and added to by the later ones.  Save and
 * recompute give the same bits.  Needs ffn_fp8 = 0 and reduce_dense = 0.
 *   x, dout [T, H] cfg->dtype; topk_idx, topk_w, keep: the forward's (saved).
 *   ws: moe_backward_workspace_bytes(cfg) bytes (one chunk slot of receive-row
 *   buffers and the fp32 slot gradients), zero-filled once before first use.
 */
size_t moe_backward_workspace_bytes(const moe_config *cfg);
moe_status moe_layer_backward(const moe_config *cfg, const void *x, const void *dout,
                              const void *w13, const void *w2, const void *w13_shared,
                              const void *w2_shared, const int32_t *topk_idx, const float *topk_w,
                              const uint8_t *keep, const void *xr_saved, const void *y_saved,
                              void *dx, float *dlogits, float *dbias, float *dw13, float *dw2,
                              float *dw13_shared, float *dw2_shared, int32_t accumulate, void *ws,
                              cudaStream_t stream);

/*
 * moe_forward_chunked with the activations in HOST memory: what a caller whose
 * tokens arrive from the host calls.  The weights stay device-resident.
 *   logits_host [T, E] float, bias_host [E] float or NULL, x_host [T, H]
 *            cfg->dtype: read by host-to-device copies into the workspace.
 *   out_host [T, H] cfg->dtype: written by device-to-host copies, chunk by
 *            chunk as each chunk's combine finishes.
 *   w13, w2, w13_shared, w2_shared, w13_scale, w2_scale, topk_idx, topk_w,
 *            keep, splits_host: as in moe_forward_chunked (device pointers but
 *            for splits_host).
 *   ws: moe_forward_host_workspace_bytes(cfg) bytes (the forward workspace
 *            plus staging for logits, bias, x and out).
 * Ordering: logits and bias are copied on s_dispatch ahead of routing; chunk
 * c's rows of x on s_compute, overlapping routing; chunk c's output on
 * s_dispatch behind chunk c+1's dispatch, overlapping chunk c+1's FFN.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for
 * the copies to be asynchronous; pageable ones work but the copies then block
 * the host.  The caller must leave the inputs unchanged and must not read
 * out_host until both streams have passed the call (e.g. synchronise
 * s_dispatch).  The result equals moe_forward_chunked's bit for bit (with
 * reduce_dense = 1 up to the order of the fp32 atomic additions, which varies
 * from run to run in both).
 */
size_t moe_forward_host_workspace_bytes(const moe_config *cfg);
moe_status moe_forward_host(const moe_config *cfg, const float *logits_host,
                            const float *bias_host, const void *x_host, const void *w13,
                            const void *w2, const void *w13_shared, const void *w2_shared,
                            const uint8_t *w13_scale, const uint8_t *w2_scale,
                            void *out_host, int32_t *topk_idx, float *topk_w, uint8_t *keep,
                            int32_t *splits_host, void *ws,
                            cudaStream_t s_dispatch, cudaStream_t s_compute);

/*
 * Watchdog self-test (failure detection; no counterpart on the pages): runs the
 * library's own bounded-wait code on something that never completes, with a
 * short limit, so a caller can check that a wait that runs out is reported and
 * that the context stays usable.
 *   which 0: the FFN's cluster-scope mbarrier wait (slice queue, scale ring) on a
 *            barrier nothing arrives at;
 *   which 1: the FFN's CTA-scope mbarrier wait (operand ring, accumulators) on a
 *            barrier nothing arrives at.
 *   limit_us in [1, 2000000].
 * One thread waits about limit_us, sets MOE_DEV_WAIT_TIMEOUT in ws's status word
 * and returns; read it with moe_device_status.  ws: moe_workspace_bytes(cfg).
 */
moe_status moe_watchdog_selftest(const moe_config *cfg, int32_t which, int32_t limit_us,
                                 void *ws, cudaStream_t stream);

/* Expert-parallel exchange, receive side: regroup the rows one rank received from
 * the other ranks of its EP group (axolotl docs, integrations.expert_parallel.args:
 * expert_parallel_backend = torch, all_to_all_single over the EP group).
 *
 * With experts owned by contiguous blocks of E / ep per rank and tokens by
 * contiguous blocks per source rank, a rank that sent each destination the rows of
 * that destination's experts in its own (expert, token) order (rows
 * [rank_offsets[d], rank_offsets[d+1]) of moe_dispatch_layout, permuted by
 * moe_permute) receives, after a variable all-to-all, cells (s, e) - the rows
 * source rank s sent for this rank's local expert e - source after source, each
 * source's cells in expert order.  The grouped FFN wants them expert after expert;
 * (expert, source, token) is then the (expert, token) order of the whole group.
 *
 *   inverse = 0: in  source-major (rows [src_off(s, e), +counts[s][e]) per cell),
 *                out expert-major (expert e's rows from sources 0, 1, ... in turn);
 *   inverse = 1: in  expert-major (the FFN's outputs), out source-major (for the
 *                reverse all-to-all).
 * counts: device int32 [ep][E / ep], counts[s][e] = rows of cell (s, e); their sum
 * must be `rows` (else MOE_DEV_BAD_INDEX is set in ws's status word and nothing is
 * read or written past `rows`).  in, out: [rows, H] in the layer dtype (bf16 or
 * fp32; cfg->ffn_fp8 = 0), 16-byte aligned, distinct.  expert_offsets (device
 * int32 [E / ep + 1], or NULL): written with the expert-major buffer's offsets of
 * each local expert (the grouped FFN's expert_offsets for these rows; all zero when
 * rows = 0).  cfg: ep = the EP group's size, E its experts.
 * ws: moe_workspace_bytes(cfg). */
moe_status moe_ep_regroup(const moe_config *cfg, const int32_t *counts, const void *in, void *out,
                          int64_t rows, int32_t inverse, int32_t *expert_offsets, void *ws,
                          cudaStream_t stream);

/* Synchronises `stream`, copies the device status word of ws to *flags and
 * clears it.  Returns MOE_ERR_DEVICE if any bit was set. */
moe_status moe_device_status(void *ws, uint32_t *flags, cudaStream_t stream);

/* Static description of a status code. */
const char *moe_status_string(moe_status status);

/* Message for the calling thread's last non-OK status ("" if none). */
const char *moe_last_error_detail(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
