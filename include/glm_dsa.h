/*
 * glm_dsa.h -- C ABI of the GLM-5.3-Flash kpool DSA decode hot path on B200 (sm_100a).
 *
 * The path, in the order the pages give it:
 *   glm_kv_store_int8      -> 528-byte int8 latent cache rows
 *   glm_kpool_build        -> k_norm LayerNorm + slot-axis softmax pooling into fp32 pooled keys
 *   glm_index_scores_topk  -> relu head-weighted index scores and the top select_k pools
 *   glm_expand_selection   -> token indices (+ cache rows), visible tail, -1 padding
 *   (glm_index_topk_expand -> the two above in one launch)
 *   (glm_dsa_decode_step   -> the whole step in one call)
 *   glm_sparse_mla_decode  -> sparse NoPE MLA over the gathered int8 rows (split-KV + combine)
 *
 * Conventions for every entry point
 *   - Pointers named *_dev are device pointers on the current CUDA device; everything else is
 *     host memory. The caller owns every buffer; the library allocates nothing, keeps no state
 *     between calls and only enqueues work on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Outputs are valid once the stream has reached the call.
 *   - Device pointers must be 16-byte aligned; leading dimensions are in elements.
 *   - Arguments are checked on the host before anything is enqueued. A failed check returns a
 *     negative status and enqueues nothing. GLM_ERR_CUDA means a launch failed (the status of
 *     cudaGetLastError is reported through glm_last_cuda_error()).
 *   - Every output element an entry point documents is written (no uninitialised tails).
 *   - Kernels never trap and never read outside the buffers described here: an index outside
 *     the documented range is treated as padding (-1) instead of being dereferenced.
 */
#ifndef GLM_DSA_H
#define GLM_DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------------------------------ */
/* Status codes                                                                                */
/* ------------------------------------------------------------------------------------------ */
#define GLM_OK 0
#define GLM_ERR_INVALID_ARG (-1) /* null / misaligned pointer, bad size or leading dimension   */
#define GLM_ERR_UNSUPPORTED (-2) /* geometry other than the one the kernels are built for      */
#define GLM_ERR_WORKSPACE (-3)   /* workspace null or smaller than glm_dsa_workspace_size()    */
#define GLM_ERR_CUDA (-4)        /* a kernel launch failed                                     */

/* latent cache row formats (glm_dsa_step.cache_format) */
#define GLM_CACHE_INT8 0         /* int8 codes, fp32 row scale, 528 bytes (glm_kv_store_int8)  */
#define GLM_CACHE_FP8 1          /* E4M3 codes, fp32 row scale, 528 bytes (glm_kv_store_fp8)   */
#define GLM_CACHE_FP4 2          /* E2M1 codes, E4M3 scale per 16, fp32 row scale, 304 bytes   */

/* Sentinel of an unused index entry ("Module glm5next_dsa_ref": INVALID). */
#define GLM_INVALID (-1)

/* Bytes of one cache row: 512 int8 codes, one little-endian fp32 scale, 12 zero bytes
 * ("GLM-5.3 Kernels" README, 'Included': titan_kv.store_int8). */
#define GLM_ROW_BYTES 528

/*
 * Geometry of one sparse-attention layer ("Module glm5next_dsa_ref": DsaDims, read from the
 * config and never defaulted; "GLM-5.3-Flash" pypto-lib page, 'Checkpoint shape').
 * The kernels are built for kv_lora_rank 512, qk_rope_head_dim 0 (NoPE: the rope slice is
 * zero-width), index_n_heads 32, index_head_dim 128, index_kpool 4, 1 <= n_heads <= 128.
 * Any other value gives GLM_ERR_UNSUPPORTED; index_topk is informational (select_k is passed
 * per call) but must be a positive multiple of index_kpool.
 */
typedef struct glm_dsa_dims {
    int32_t kv_lora_rank;
    int32_t qk_rope_head_dim;
    int32_t n_heads;
    int32_t index_n_heads;
    int32_t index_head_dim;
    int32_t index_kpool;
    int32_t index_topk;
} glm_dsa_dims;

/* Returns GLM_OK if `dims` is the geometry the kernels implement. */
int glm_check_dims(const glm_dsa_dims *dims);

/* Human-readable name of a status code (static storage). */
const char *glm_status_string(int status);

/* cudaError_t value of the last launch that returned GLM_ERR_CUDA on this host thread. */
int glm_last_cuda_error(void);

/* ------------------------------------------------------------------------------------------ */
/* store_int8                                                                                  */
/* ------------------------------------------------------------------------------------------ */
/*
 * "GLM-5.3 Kernels" README, 'Included' (titan_kv.store_int8): quantise each 512-value BF16 MLA
 * latent into one 528-byte cache row -- bytes [0,512) int8 codes, [512,516) fp32 scale
 * (little endian), [516,528) zero -- and scatter it to row slots[i]; slots[i] < 0 is padding
 * and writes nothing. scale = max(amax, 1e-4f) / 127 (fp32), code = clamp(rint(x / scale), +-127)
 * with an IEEE fp32 quotient and ties to even.
 *   latent_dev  bf16 [n, 512], rows contiguous (row stride 1024 bytes)
 *   slots_dev   int64 [n]
 *   cache_dev   int8 [n_rows, 528] (rows contiguous; blocks of 256 rows are just consecutive rows)
 * A slot >= n_rows is outside the contract and is skipped. Duplicate slots race (last writer
 * undefined). n == 0 is a no-op.
 */
int glm_kv_store_int8(const glm_dsa_dims *dims, const void *latent_dev, const int64_t *slots_dev,
                      int64_t n, int8_t *cache_dev, int64_t n_rows, void *stream);

/*
 * The FP8 latent cache ("GLM on CUDA": an opt-in FP8 latent cache, --kv-dtype fp8, lossy; the
 * page gives no format). The row of glm_kv_store_int8 with E4M3 codes (OCP E4M3FN: exponent bias
 * 7, subnormals, largest finite 448) in bytes [0,512): scale = max(amax, 1e-4f) / 448 (fp32), code =
 * the E4M3 value nearest the IEEE fp32 quotient x / scale, ties to the even code, saturating at
 * +-448, the sign kept. Arguments, slots and padding as glm_kv_store_int8; cache_dev uint8 [n_rows, 528].
 */
int glm_kv_store_fp8(const glm_dsa_dims *dims, const void *latent_dev, const int64_t *slots_dev,
                     int64_t n, uint8_t *cache_dev, int64_t n_rows, void *stream);

/*
 * The 4-bit latent cache ("GLM on CUDA": an opt-in 4-bit latent cache, --kv-dtype fp4, lossy; the
 * page gives no format). A 304-byte row of E2M1 codes (sign, 2 exponent bits with bias 1, 1
 * mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) with one E4M3 scale per 16 values and one
 * fp32 scale per row:
 *   s_row = max(amax, 1e-4f) / 2688          (2688 = 6 * 448)
 *   e_k   = E4M3(bmax_k / (6 * s_row))       (bmax_k: largest |x| of values 16k .. 16k+15)
 *   d_k   = value(e_k) * s_row
 *   code  = E2M1(x / d_k), 0 where d_k == 0
 * each an IEEE fp32 operation; E4M3() and E2M1() round to the nearest value, ties to the even
 * code, saturating (448, 6), the sign kept. Bytes [0,256): code pairs (byte i: value 2i in the low
 * nibble, 2i+1 in the high nibble); [256,288): e_0 .. e_31; [288,292): s_row (little endian);
 * [292,304): zeros. The value of an entry is value(code) * value(e_k) * s_row. Arguments, slots
 * and padding as glm_kv_store_int8; cache_dev uint8 [n_rows, 304] (16-byte aligned).
 */
int glm_kv_store_fp4(const glm_dsa_dims *dims, const void *latent_dev, const int64_t *slots_dev,
                     int64_t n, uint8_t *cache_dev, int64_t n_rows, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* kpool_build                                                                                 */
/* ------------------------------------------------------------------------------------------ */
/*
 * "Module glm5next_dsa_ref", pool_states and its traps: k is normalised by k_norm (a LayerNorm
 * with bias over the 128 channels, eps = ln_eps); pool p of sequence b covers the kpool = 4
 * tokens t_s = pad[b] + 4p + s (pooling starts at the first valid token); a pool exists only if
 * all 4 slots are valid tokens (p < len[b] / 4); the 4 slots are mixed per channel by a softmax
 * of the gates over the slot axis:
 *     pooled[b][p][d] = sum_s softmax_s(gate[b][t_s][d]) * LN(k[b][t_s])[d]      (fp32)
 *   k_dev, gate_dev  bf16 [batch, ld_tokens, 128]: token t of sequence b at row b*ld_tokens + t
 *                    (padded coordinates; positions < pad[b] are padding and never read)
 *   ln_w_dev, ln_b_dev  fp32 [128]
 *   pad_dev, len_dev    int32 [batch]: first valid position and valid length of each sequence
 *   pool_begin_dev      int32 [batch] or NULL (= 0): first pool to (re)build per sequence
 *   max_new_pools       pools built per sequence: p in [pool_begin, min(pool_begin +
 *                       max_new_pools, len/4, ld_pools)); e.g. 1 for a decode step
 *   pooled_dev          fp32 [batch, ld_pools, 128]; pools outside that range are not touched
 *   n_pools_dev         int32 [batch] or NULL: receives len[b] / 4 (capped at ld_pools)
 * Requires pad[b] + len[b] <= ld_tokens (not checked on the device: rows past it are not read).
 */
int glm_kpool_build(const glm_dsa_dims *dims, const void *k_dev, const void *gate_dev,
                    int64_t ld_tokens, const float *ln_w_dev, const float *ln_b_dev, float ln_eps,
                    const int32_t *pad_dev, const int32_t *len_dev, const int32_t *pool_begin_dev,
                    int32_t batch, int32_t max_new_pools, float *pooled_dev, int64_t ld_pools,
                    int32_t *n_pools_dev, void *stream);

/*
 * The INT8 indexer state ("GLM-5.3-Flash" pypto-lib page, 'What is quantized': the indexer state
 * cache is FP32 today; the sibling port keeps it in INT8 with one FP32 scale per row). The same
 * pools as glm_kpool_build, each stored as 128 int8 codes and one fp32 scale instead of 128 fp32
 * values: scale = max(amax, 1e-4f) / 127 over the pool's fp32 key, code = clamp(rint(x / scale),
 * +-127) with an IEEE fp32 quotient and ties to even (the recipe of the latent cache rows).
 *   pooled_codes_dev   int8 [batch, ld_pools, 128] (16-byte aligned)
 *   pooled_scales_dev  fp32 [batch, ld_pools]
 * Everything else as glm_kpool_build.
 */
int glm_kpool_build_q8(const glm_dsa_dims *dims, const void *k_dev, const void *gate_dev,
                       int64_t ld_tokens, const float *ln_w_dev, const float *ln_b_dev, float ln_eps,
                       const int32_t *pad_dev, const int32_t *len_dev, const int32_t *pool_begin_dev,
                       int32_t batch, int32_t max_new_pools, int8_t *pooled_codes_dev,
                       float *pooled_scales_dev, int64_t ld_pools, int32_t *n_pools_dev, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* index_scores + topk_pools                                                                   */
/* ------------------------------------------------------------------------------------------ */
/*
 * "Module glm5next_dsa_ref", index_scores (matmul -> relu -> head-weighted sum) and topk_pools.
 * For query n of sequence b = q_seq[n] at padded position q_pos[n], the visible pools are the
 * existing pools whose 4 slots are all visible (causal, not padding):
 *     n_vis = min(len[b] / 4, max(0, q_pos - pad[b] + 1) / 4, ld_pools)
 *     score[n][p] = sum_h w[n][h] * max(0, sum_d q_idx[n][h][d] * pooled[b][p][d]),  p < n_vis
 * and the selection is the min(select_k, n_vis) highest scores, ordered by score descending
 * with ties to the lower pool id (-0.0 == +0.0), followed by -1 up to select_k.
 *   q_idx_dev   bf16 [n_q, 32, 128]        w_dev  fp32 [n_q, 32]
 *   pooled_dev  fp32 [batch, ld_pools, 128] (from glm_kpool_build)
 *   q_seq_dev, q_pos_dev  int32 [n_q];     pad_dev, len_dev  int32 [batch]
 *   scores_dev  fp32 [n_q, ld_pools] or NULL: receives the scores (entries p >= n_vis are -inf)
 *   topk_dev    int32 [n_q, select_k]      n_sel_dev  int32 [n_q] or NULL
 *   workspace_dev / ws_bytes: >= glm_dsa_workspace_size(dims, GLM_OP_INDEX_SCORES_TOPK, ...), 256-byte
 *               aligned (required even when scores_dev is given; contents on entry are ignored).
 *               Its last 256 bytes start with a status word set nonzero if a wait gave up (on the
 *               tensor cores, or of the CTAs of one query for one another); the outputs are then
 *               invalid. The library never clears it.
 * 1 <= select_k <= 2048. The q . pooled products run on the tensor cores: each (query, head) is
 * scaled by a power of two and taken exactly as fp16; each fp32 pooled key is scaled by a power
 * of two and split into two fp16 terms (together the key to 2^-22 of its largest element), so the
 * dot products carry that and fp32 accumulation error only (relative error far below 1e-4); relu
 * and the head weights in fp32.
 * Fewer than 128 queries: one fused launch (scores, selection, expansion), one or more CTAs per
 * query streaming its visible pools. 128 queries or more (fp32 keys): the many-query path -- a
 * query preparation kernel, a scoring kernel whose CTAs each convert 256 pooled keys once for
 * every query of their sequence (pools on the MMA M dimension, 4 queries x 32 heads on N), then
 * the selection of glm_topk_pools on those scores (and the expansion): five launches, the same
 * outputs under the same rules; the workspace then also holds the queries as fp16 (8 KB each).
 */
int glm_index_scores_topk(const glm_dsa_dims *dims, const void *q_idx_dev, const float *w_dev,
                          const float *pooled_dev, int64_t ld_pools, const int32_t *q_seq_dev,
                          const int32_t *q_pos_dev, const int32_t *pad_dev, const int32_t *len_dev,
                          int32_t batch, int32_t n_q, int32_t select_k, float *scores_dev,
                          int32_t *topk_dev, int32_t *n_sel_dev, void *workspace_dev,
                          size_t ws_bytes, void *stream);

/*
 * glm_index_scores_topk followed by glm_expand_selection, in one launch (fewer than 128 queries;
 * else the many-query path of glm_index_scores_topk, then the expansion): the same scores, top-k
 * row and n_sel, plus the expansion of the selection into token positions and cache rows
 * ("Module glm5next_dsa_ref", expand_selection; the rules and arguments of glm_expand_selection:
 * slot_map_dev int64 [batch, ld_slot] or NULL, tok_dev / rows_dev int32 [n_q, out_width], at
 * least one of them non-NULL, out_width >= 4 * select_k + 3). Every output equals what the two
 * separate calls produce. The workspace is that of GLM_OP_INDEX_SCORES_TOPK.
 * When the selection of a query spans several CTAs they meet at a grid barrier: the launch sizes
 * its grid to at most one CTA per SM and needs every CTA resident at once (a GPU shared with
 * other concurrent work that holds SMs indefinitely breaks that); a wait that gives up sets the
 * status word nonzero and leaves the outputs invalid.
 */
int glm_index_topk_expand(const glm_dsa_dims *dims, const void *q_idx_dev, const float *w_dev,
                          const float *pooled_dev, int64_t ld_pools, const int32_t *q_seq_dev,
                          const int32_t *q_pos_dev, const int32_t *pad_dev, const int32_t *len_dev,
                          int32_t batch, int32_t n_q, int32_t select_k, const int64_t *slot_map_dev,
                          int64_t ld_slot, int32_t out_width, float *scores_dev, int32_t *topk_dev,
                          int32_t *n_sel_dev, int32_t *tok_dev, int32_t *rows_dev, void *workspace_dev,
                          size_t ws_bytes, void *stream);

/*
 * glm_index_topk_expand on the INT8 indexer state (glm_kpool_build_q8): each pooled key is
 * code * scale, so score[n][p] = scale[p] * sum_h w[n][h] * max(0, sum_d q_idx[n][h][d] * code[p][d])
 * (relu commutes with the positive scale). The codes are exact in bf16, so the products carry
 * fp32 accumulation error only. Arguments, outputs and workspace as glm_index_topk_expand.
 */
int glm_index_topk_expand_q8(const glm_dsa_dims *dims, const void *q_idx_dev, const float *w_dev,
                             const int8_t *pooled_codes_dev, const float *pooled_scales_dev,
                             int64_t ld_pools, const int32_t *q_seq_dev, const int32_t *q_pos_dev,
                             const int32_t *pad_dev, const int32_t *len_dev, int32_t batch, int32_t n_q,
                             int32_t select_k, const int64_t *slot_map_dev, int64_t ld_slot,
                             int32_t out_width, float *scores_dev, int32_t *topk_dev, int32_t *n_sel_dev,
                             int32_t *tok_dev, int32_t *rows_dev, void *workspace_dev, size_t ws_bytes,
                             void *stream);

/*
 * The scores alone ("Module glm5next_dsa_ref", index_scores): the same scores as
 * glm_index_scores_topk, written to scores_dev fp32 [n_q, ld_pools] (entries p >= n_vis are
 * -inf), without the selection. No workspace.
 */
int glm_index_scores(const glm_dsa_dims *dims, const void *q_idx_dev, const float *w_dev,
                     const float *pooled_dev, int64_t ld_pools, const int32_t *q_seq_dev,
                     const int32_t *q_pos_dev, const int32_t *pad_dev, const int32_t *len_dev,
                     int32_t batch, int32_t n_q, float *scores_dev, void *stream);

/*
 * The selection alone, on given scores ("Module glm5next_dsa_ref", topk_pools): for each query
 * n, the min(select_k, n_visible[n]) highest of scores[n][0 .. n_visible[n]) in the order above,
 * then -1. Used to check the selection bit-exactly on externally supplied scores.
 *   scores_dev  fp32 [n_q, ld_scores];  n_visible_dev int32 [n_q] (clamped to [0, ld_scores])
 *   topk_dev    int32 [n_q, select_k];  n_sel_dev int32 [n_q] or NULL
 *   workspace_dev / ws_bytes: >= glm_dsa_workspace_size(dims, GLM_OP_TOPK_POOLS, n_q, ld_scores, ...),
 *               256-byte aligned; contents on entry are ignored
 * NaN scores are outside the contract.
 */
int glm_topk_pools(const float *scores_dev, int64_t ld_scores, const int32_t *n_visible_dev,
                   int32_t n_q, int32_t select_k, int32_t *topk_dev, int32_t *n_sel_dev,
                   void *workspace_dev, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* expand_selection                                                                            */
/* ------------------------------------------------------------------------------------------ */
/*
 * "Module glm5next_dsa_ref", expand_selection and the -1 trap: each selected pool p (in top-k
 * order) becomes its 4 tokens pad + 4p + 0..3; then the visible tail (tokens pad + 4*n_vis ..
 * q_pos, at most 3); then -1 up to out_width. Every one of the out_width entries is written.
 *   topk_dev     int32 [n_q, select_k] (-1 ends the list; entries >= n_vis are treated as -1)
 *   n_sel_dev    int32 [n_q] or NULL (NULL: the list ends at the first -1)
 *   slot_map_dev int64 [batch, ld_slot] or NULL: cache row of token t of sequence b, -1 if none
 *   tok_dev      int32 [n_q, out_width] or NULL: token positions
 *   rows_dev     int32 [n_q, out_width] or NULL: cache rows (slot_map[b][tok]; tok itself when
 *                slot_map is NULL); -1 where the token is -1 or has no row
 * Requires out_width >= 4 * select_k + 3 (the largest possible selection plus a full tail).
 */
int glm_expand_selection(const glm_dsa_dims *dims, const int32_t *topk_dev,
                         const int32_t *n_sel_dev, const int32_t *q_seq_dev,
                         const int32_t *q_pos_dev, const int32_t *pad_dev, const int32_t *len_dev,
                         int32_t batch, int32_t n_q, int32_t select_k,
                         const int64_t *slot_map_dev, int64_t ld_slot, int32_t out_width,
                         int32_t *tok_dev, int32_t *rows_dev, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* sparse NoPE MLA decode                                                                      */
/* ------------------------------------------------------------------------------------------ */
/*
 * "GLM-5.3 Kernels" README, 'Included' (titan_mla.triton_mla_sparse_attention) and 'The tested
 * MLA contract': int8 rows are dequantised in-kernel (c = code * scale) and the shared 512-d
 * latent is both K and V (one KV head, NoPE); softmax and accumulation in fp32:
 *     s[h][j] = sm_scale * q[n][h] . c_j,  out[n][h] = sum_j softmax_j(s[h])_j c_j,
 *     lse[n][h] = log sum_j exp(s[h][j])
 * over the entries j of rows[n] with 0 <= rows[n][j] < n_rows (each entry is one key; -1 is
 * padding). A query with no valid entry gets out = 0 and lse = -inf. Split-KV: chunks of the
 * index row run in parallel and a combine kernel merges their partial softmax states.
 *   q_dev      bf16 [n_q, n_heads, 512]       cache_dev int8 [n_rows, 528]
 *   rows_dev   int32 [n_q, width]             out_dev   bf16 [n_q, n_heads, 512]
 *   lse_dev    fp32 [n_q, n_heads] or NULL    out_f32_dev fp32 [n_q, n_heads, 512] or NULL
 *   workspace_dev / ws_bytes: >= glm_dsa_workspace_size(dims, GLM_OP_SPARSE_MLA, n_q, 0, 0, width),
 *               256-byte aligned. Its last 256 bytes start with a status word that the kernels set
 *               nonzero if a wait on the tensor cores gave up (the outputs are then invalid); it is
 *               never cleared by the library, so a caller that checks it zeroes it first.
 * 1 <= width <= 65536. The contractions run on the tensor cores with fp16 operands, accumulating
 * in fp32: the int8 codes exactly, each query head exactly after scaling it by a power of two
 * (values below 2^-17 of the head's scaled range aside), the softmax weights as a two-term fp16
 * split of p * scale_row / (the chunk's largest row scale).
 */
int glm_sparse_mla_decode(const glm_dsa_dims *dims, const void *q_dev, const int8_t *cache_dev,
                          int64_t n_rows, const int32_t *rows_dev, int32_t n_q, int32_t width,
                          float sm_scale, void *out_dev, float *lse_dev, float *out_f32_dev,
                          void *workspace_dev, size_t ws_bytes, void *stream);

/*
 * glm_sparse_mla_decode over FP8 rows (glm_kv_store_fp8): each entry's key and value is
 * value(code) * scale, the E4M3 codes widened to bf16 exactly; everything else as
 * glm_sparse_mla_decode (cache_dev uint8 [n_rows, 528], same workspace).
 */
int glm_sparse_mla_decode_fp8(const glm_dsa_dims *dims, const void *q_dev, const uint8_t *cache_dev,
                              int64_t n_rows, const int32_t *rows_dev, int32_t n_q, int32_t width,
                              float sm_scale, void *out_dev, float *lse_dev, float *out_f32_dev,
                              void *workspace_dev, size_t ws_bytes, void *stream);

/*
 * glm_sparse_mla_decode over 4-bit rows (glm_kv_store_fp4): each entry's key and value is
 * value(code) * value(e_k) * s_row; code * block scale is widened to fp16 exactly (a product of
 * magnitude in [2^-10, 2688] with at most 6 significant bits) and s_row is applied as the INT8
 * row's scale is; everything else as glm_sparse_mla_decode (cache_dev uint8 [n_rows, 304], same
 * workspace).
 */
int glm_sparse_mla_decode_fp4(const glm_dsa_dims *dims, const void *q_dev, const uint8_t *cache_dev,
                              int64_t n_rows, const int32_t *rows_dev, int32_t n_q, int32_t width,
                              float sm_scale, void *out_dev, float *lse_dev, float *out_f32_dev,
                              void *workspace_dev, size_t ws_bytes, void *stream);

/*
 * The same sparse NoPE MLA decode without a workspace argument. The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory where they run the
 * attention -- plugin interfaces that pass a kernel only its inputs and outputs, and serving
 * loops that allow no allocation after start-up. Arguments, results and checks are those of
 * glm_sparse_mla_decode minus the workspace; the split partials live instead in one fixed
 * scratch array of GLM_NOALLOC_SCRATCH_BYTES compiled into the library (held on every GPU that
 * loads the library until the process exits). This call itself allocates nothing.
 *   - A request needing more than the scratch holds -- n_q * ceil(width / 64) * n_heads partials of
 *     2,056 bytes each, each region rounded up to 256 bytes, plus 256 bytes -- returns
 *     GLM_ERR_WORKSPACE before anything is enqueued (one 64-head query of width 2,176 needs about
 *     4.5 MiB, one 128-head query about 9 MiB).
 *   - Every call looks up the scratch's device address on the device current at the call; the
 *     first call on a device also loads the library's device code there, so make that first call
 *     before any stream capture.
 *   - Every call shares the one array, and the status word is cleared at the start of each call:
 *     calls that overlap on the GPU (other streams, other host threads) race on it and must be
 *     serialised by the caller.
 *   - The caller cannot read the scratch's status word; if a wait on the tensor cores gave up, the
 *     call's outputs (out, lse, out_f32) are NaN instead.
 */
#define GLM_NOALLOC_SCRATCH_BYTES (16u << 20)
int glm_sparse_mla_decode_noalloc(const glm_dsa_dims *dims, const void *q_dev,
                                  const int8_t *cache_dev, int64_t n_rows, const int32_t *rows_dev,
                                  int32_t n_q, int32_t width, float sm_scale, void *out_dev,
                                  float *lse_dev, float *out_f32_dev, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* up-projection of the attention output                                                       */
/* ------------------------------------------------------------------------------------------ */
/*
 * "Module glm5next_dsa_ref", expand_kv (kv_b_proj maps the 512-d latent to per-head K and V) and
 * "GLM-5.3-Flash" pypto-lib page, 'Checkpoint shape' (qk_head_dim / v_head_dim 256) and 'Open
 * questions an owner will hit' (kv_b_proj is BF16): the latent-space attention output of each head
 * taken to that head's value space,
 *     out_v[n][h][e] = sum_d o_lat[n][h][d] * W[h (dk + dv) + dk + e][d],   e < dv, d < 512,
 * which with the absorbed query (q_lat[h] = W_K,h^T q_h) equals attention over the expanded K and V.
 *   o_lat_dev    bf16 [n_q, n_heads, 512]   (the out_dev of glm_sparse_mla_decode)
 *   w_kv_b_dev   bf16 [n_heads * (dk + dv), 512], torch Linear layout: per head dk K rows, then dv V rows
 *   out_v_dev    bf16 [n_q, n_heads, dv]    out_v_f32_dev fp32 [n_q, n_heads, dv] or NULL
 * dk = qk_nope_head_dim >= 0, dv = v_head_dim a multiple of 128 (<= 4096). Pointers 16-byte aligned.
 * Tensor cores (bf16 operands, fp32 accumulation); W is read once per 128 queries. If a bounded wait
 * gives up, the affected outputs are NaN. Returns GLM_OK, GLM_ERR_INVALID_ARG / _UNSUPPORTED (before
 * anything is enqueued) or GLM_ERR_CUDA.
 */
int glm_mla_v_up(const glm_dsa_dims *dims, const void *o_lat_dev, const void *w_kv_b_dev,
                 int32_t qk_nope_head_dim, int32_t v_head_dim, int32_t n_q, void *out_v_dev,
                 float *out_v_f32_dev, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* context parallelism: one sequence's pools and rows over several ranks                        */
/* ------------------------------------------------------------------------------------------ */
/*
 * TensorFold issue #402, 'Credit': tokens are interleaved over the ranks, local candidates are
 * merged into the global top-k, and attention partials are merged by log-sum-exp in rank order.
 * Here the unit is the pool: rank r of `world` holds the pools p = r + world i (stored at local
 * index i, with the cache rows of their tokens) and the visible tail when it would own the next
 * pool. Each rank selects its local top-k (glm_index_scores_topk, keeping the scores), turns it into
 * (score, global pool id) candidates, the ranks exchange them (a collective of the caller's), and
 * every rank runs the same merge, which equals the selection over all pools; each rank then
 * attends over the selected rows it holds and the ranks exchange and merge those results.
 *
 * glm_cp_candidates: cand_scores[n][x] = scores[n][topk[n][x]], cand_ids[n][x] = topk[n][x] * world
 *   + rank (-1 where topk is -1 or past ld_scores).  scores fp32 [n_q, ld_scores], topk int32
 *   [n_q, select_k] (local indices), cand_* [n_q, select_k].
 * glm_merge_topk: over the candidates of n_parts parts, laid out [n_parts][n_q][per_part] (what an
 *   all-gather of every rank's [n_q][per_part] arrays gives), the select_k best (score descending,
 *   then the lower id; ids must be distinct) per query into topk [n_q, select_k] (-1 padded) and
 *   n_sel [n_q] (or NULL).
 * glm_lse_merge: out_parts fp32 [n_parts][n_q][n_heads][512] (normalised attention outputs over
 *   disjoint row sets) and lse_parts fp32 [n_parts][n_q][n_heads] -> LSE = log sum_r e^{lse_r},
 *   out = sum_r e^{lse_r - LSE} out_r (bf16 [n_q][n_heads][512], fp32 copy and lse optional),
 *   parts taken in order; a part with lse = -inf contributes nothing.
 * All return GLM_OK, GLM_ERR_INVALID_ARG (before anything is enqueued) or GLM_ERR_CUDA.
 */
int glm_cp_candidates(const float *scores_dev, int64_t ld_scores, const int32_t *topk_dev, int32_t n_q,
                      int32_t select_k, int32_t rank, int32_t world, float *cand_scores_dev,
                      int32_t *cand_ids_dev, void *stream);
int glm_merge_topk(const float *cand_scores_dev, const int32_t *cand_ids_dev, int32_t n_parts, int32_t n_q,
                   int32_t per_part, int32_t select_k, int32_t *topk_dev, int32_t *n_sel_dev, void *stream);
int glm_lse_merge(const glm_dsa_dims *dims, const float *out_parts_dev, const float *lse_parts_dev,
                  int32_t n_parts, int32_t n_q, void *out_dev, float *out_f32_dev, float *lse_dev, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* testing                                                                                    */
/* ------------------------------------------------------------------------------------------ */
/*
 * The number of polls after which a wait of the fused index kernel's CTAs on one another (the
 * sample meeting, the candidate meeting) gives up, on the current device: GLM_CROSS_CTA_WAIT_LIMIT
 * by default. A test lowers it (0: every such wait gives up at once) to check the give-up path
 * without a fault: the kernel sets bit 8 of the status word, leaves its selection outputs
 * unwritten and returns; restore the default afterwards. Not for use while kernels of the
 * library run on the device. Returns GLM_OK or GLM_ERR_CUDA.
 */
#define GLM_CROSS_CTA_WAIT_LIMIT (1u << 21)
int glm_debug_set_cross_cta_wait_limit(uint32_t polls);

/* ------------------------------------------------------------------------------------------ */
/* the whole decode step in one call                                                           */
/* ------------------------------------------------------------------------------------------ */
/*
 * Arguments of glm_dsa_decode_step: those of glm_kv_store_int8, glm_kpool_build,
 * glm_index_topk_expand and glm_sparse_mla_decode (same names, meanings, layouts and rules; the
 * cache rows written by the store are the rows the attention reads, so slot_map_dev must map the
 * new tokens to the slots in slots_dev). Every pointer is a device pointer.
 */
typedef struct glm_dsa_step {
    /* store_int8: n_new new latent rows */
    const void *latent_dev;        /* bf16 [n_new, 512]                  */
    const int64_t *slots_dev;      /* int64 [n_new]                      */
    int64_t n_new;
    int8_t *cache_dev;             /* int8 [n_rows, 528]                 */
    int64_t n_rows;
    /* kpool_build: up to max_new_pools new pools per sequence from pool_begin_dev */
    const void *k_dev;             /* bf16 [batch, ld_tokens, 128]       */
    const void *gate_dev;          /* bf16 [batch, ld_tokens, 128]       */
    int64_t ld_tokens;
    const float *ln_w_dev;         /* fp32 [128]                         */
    const float *ln_b_dev;         /* fp32 [128]                         */
    float ln_eps;
    const int32_t *pad_dev;        /* int32 [batch]                      */
    const int32_t *len_dev;        /* int32 [batch]                      */
    const int32_t *pool_begin_dev; /* int32 [batch] or NULL              */
    int32_t batch;
    int32_t max_new_pools;
    float *pooled_dev;             /* fp32 [batch, ld_pools, 128]        */
    int64_t ld_pools;
    /* index scores, top-k, expansion */
    const void *q_idx_dev;         /* bf16 [n_q, 32, 128]                */
    const float *w_dev;            /* fp32 [n_q, 32]                     */
    const int32_t *q_seq_dev;      /* int32 [n_q]                        */
    const int32_t *q_pos_dev;      /* int32 [n_q]                        */
    int32_t n_q;
    int32_t select_k;
    const int64_t *slot_map_dev;   /* int64 [batch, ld_slot] or NULL     */
    int64_t ld_slot;
    int32_t out_width;             /* >= 4 * select_k + 3                */
    float *scores_dev;             /* fp32 [n_q, ld_pools] or NULL       */
    int32_t *topk_dev;             /* int32 [n_q, select_k]              */
    int32_t *n_sel_dev;            /* int32 [n_q] or NULL                */
    int32_t *tok_dev;              /* int32 [n_q, out_width] or NULL     */
    int32_t *rows_dev;             /* int32 [n_q, out_width]             */
    /* sparse MLA over rows_dev */
    const void *q_dev;             /* bf16 [n_q, n_heads, 512]           */
    float sm_scale;
    void *out_dev;                 /* bf16 [n_q, n_heads, 512]           */
    float *lse_dev;                /* fp32 [n_q, n_heads] or NULL        */
    float *out_f32_dev;            /* fp32 [n_q, n_heads, 512] or NULL   */
    /* the INT8 indexer state instead of pooled_dev (glm_kpool_build_q8), or NULL */
    int8_t *pooled_codes_dev;      /* int8 [batch, ld_pools, 128]        */
    float *pooled_scales_dev;      /* fp32 [batch, ld_pools]             */
    /* the rows of cache_dev: GLM_CACHE_INT8 (int8 [n_rows, 528]), GLM_CACHE_FP8 (uint8
     * [n_rows, 528]) or GLM_CACHE_FP4 (uint8 [n_rows, 304]); the store and the attention are those
     * of glm_kv_store_int8 / _fp8 / _fp4 and glm_sparse_mla_decode / _fp8 / _fp4. Any other value:
     * GLM_ERR_INVALID_ARG. */
    int32_t cache_format;
    /* 0: the whole step. k = 1, 2, 3: only the step's first k kernels (1: store, pool build and
     * counter zeroing; 2: + scoring, selection and expansion; 3: + the attention's split), for
     * timing a prefix of the step; the outputs of the later kernels are then not written. */
    int32_t stop_after;
} glm_dsa_step;

/*
 * One decode (or prefill-chunk) step: glm_kv_store_int8, glm_kpool_build, glm_index_topk_expand
 * and glm_sparse_mla_decode on the same stream, with the same results as those four calls in
 * that order. It runs as four kernels: the store, the pool build and the zeroing of the step's
 * counters share the first; then the fused scoring + selection + expansion; then the split and
 * the combine of the sparse attention.
 *   workspace_dev / ws_bytes: >= glm_dsa_workspace_size(dims, GLM_OP_DECODE_STEP, n_q, ld_pools,
 *               select_k, out_width), 256-byte aligned, contents on entry ignored. Its last 256
 *               bytes start with a status word set nonzero when a wait gave up (outputs invalid;
 *               never cleared by the library).
 * Checks: those of the four calls; the first failing one is returned and nothing is enqueued.
 */
int glm_dsa_decode_step(const glm_dsa_dims *dims, const glm_dsa_step *step, void *workspace_dev,
                        size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------ */
/* workspace sizes                                                                             */
/* ------------------------------------------------------------------------------------------ */
#define GLM_OP_INDEX_SCORES_TOPK 1
#define GLM_OP_TOPK_POOLS 2
#define GLM_OP_SPARSE_MLA 3
#define GLM_OP_DECODE_STEP 4

/*
 * Bytes of device workspace an entry point needs (0 if none; (size_t)-1 for bad arguments).
 *   GLM_OP_INDEX_SCORES_TOPK: n_q, max_pools = ld_pools, select_k
 *   GLM_OP_TOPK_POOLS:        n_q, max_pools = ld_scores, select_k
 *   GLM_OP_SPARSE_MLA:        n_q, width (max_pools and select_k unused)
 *   GLM_OP_DECODE_STEP:       n_q, max_pools = ld_pools, select_k, width = out_width
 */
size_t glm_dsa_workspace_size(const glm_dsa_dims *dims, int32_t op, int32_t n_q,
                              int64_t max_pools, int32_t select_k, int32_t width);

/*
 * How glm_dsa_decode_step runs a step of this shape on the current device: *launches receives
 * the number of kernels it enqueues (stop_after = 0), *paths (or NULL) a mask of
 *   GLM_PLAN_INDEX_MANY  -- 128 or more queries on fp32 keys: the many-query scoring kernel (pooled
 *                           keys shared by the queries of a sequence), then the selection and the
 *                           expansion as separate kernels; otherwise one fused index kernel;
 *   GLM_PLAN_MLA_MANY    -- enough queries to fill the SMs twice: each attention CTA walks a run
 *                           of a query's chunks; otherwise one CTA per 64-entry chunk;
 *   GLM_PLAN_MLA_COMBINE -- a combine kernel merges partials (absent when each query's entries
 *                           are covered by one CTA, which then writes the output itself).
 * int8_keys: nonzero for the INT8 indexer state. A host-side query: nothing is enqueued.
 * Returns GLM_OK, or the argument errors of glm_dsa_decode_step's shape checks.
 */
#define GLM_PLAN_INDEX_MANY 1
#define GLM_PLAN_MLA_MANY 2
#define GLM_PLAN_MLA_COMBINE 4
int glm_dsa_step_plan(const glm_dsa_dims *dims, int32_t n_q, int64_t ld_pools, int32_t batch, int32_t width,
                      int32_t int8_keys, int32_t *launches, int32_t *paths);

#ifdef __cplusplus
}
#endif

#endif /* GLM_DSA_H */
