/*
 * oracle.c -- plain, single-threaded fp64 CPU oracle of the GLM-5.3-Flash kpool DSA decode path.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's CPU
 * baseline leg may load this library. It shares no code, header, table or helper with the CUDA
 * path, and the product never calls it.
 *
 * Every function follows a passage of the pages it cites:
 *   [KERNELS]  "GLM-5.3 Kernels" README: "Included" table (titan_kv.store_int8,
 *              titan_mla.triton_mla_sparse_attention), "The tested MLA contract",
 *              "Install the standalone kernels" (cache layout and index contract).
 *   [DSA-REF]  "Module glm5next_dsa_ref": "Traps this module encodes" and the function list
 *              (layer_norm, pool_states, index_scores, topk_pools, expand_selection, visible,
 *              topk_to_mask, mla_masked_attention, kept_pools, DsaDims, INVALID).
 *   [PYPTO]    "GLM-5.3-Flash" (pypto-lib): "Checkpoint shape", "What is quantized" (incl. the
 *              INT8 indexer-state variant).
 * Where a page is silent the reading taken is stated beside the code as READING.
 *
 * Arithmetic is fp64 unless the step is an encoding fixed to fp32 (the int8 row's scale and the
 * quotient that is rounded to an int8 code), where the fp32 result is obtained exactly: an fp64
 * quotient of two fp32 values rounded once more to fp32 equals the correctly rounded fp32
 * quotient, because 53 >= 2*24 + 2.
 *
 * Parity status: every function below is pinned by the CPU test suite (closed forms, worked
 * examples of the pages, brute force on tiny inputs, invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_INVALID (-1)           /* [DSA-REF] INVALID: the invalid-index sentinel           */
#define ORACLE_ROW_BYTES 528          /* [KERNELS] 512 int8 values, one fp32 scale, 12 zero bytes */
#define ORACLE_LATENT 512             /* [PYPTO] kv_lora_rank                                     */
#define ORACLE_QMAX 127.0             /* [PYPTO] "What is quantized": rescaled to 127            */

/* READING: the amax floor is the page family's INT8_AMAX_EPS (pypto-lib "What is quantized"),
 * taken as the fp32 value nearest 1e-4 so that both sides floor with the same number. */
static double amax_floor(void) { return (double)1e-4f; }

static double bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------------------------------------
 * DsaDims check -- [DSA-REF] "DsaDims ... never defaulted" and the NoPE trap
 * ("qk_rope_head_dim = 0 ... the k_rot slice is zero-width"); [PYPTO] "the config validator
 * rejects any other value". Returns 0 when the geometry is the one the path is defined for.
 * ------------------------------------------------------------------------------------------- */
int oracle_check_dims(int kv_lora_rank, int qk_rope_head_dim, int n_heads, int index_n_heads,
                      int index_head_dim, int index_kpool)
{
    if (qk_rope_head_dim != 0) return -1;              /* NoPE: zero-width rope slice only   */
    if (kv_lora_rank != ORACLE_LATENT) return -1;      /* the latent consumed is 512 + 0 wide */
    if (n_heads <= 0 || index_n_heads <= 0 || index_head_dim <= 0 || index_kpool <= 0) return -1;
    return 0;
}

/* ---------------------------------------------------------------------------------------------
 * store_int8 -- [KERNELS] "titan_kv.store_int8": each 512-value latent becomes a 528-byte row of
 * 512 int8 values, one fp32 scale and 12 zero bytes, scattered by int64 slot; a negative slot is
 * padding and writes nothing.
 * READINGS: byte order values | scale (little endian) | zeros; scale = max(amax, floor) / 127;
 * code = clamp(round_half_even(x / scale), -127, 127) with an IEEE fp32 quotient; dequantised
 * value = code * scale.
 * Returns 0, or -1 if a slot is past the cache.
 * ------------------------------------------------------------------------------------------- */
int oracle_store_int8(const uint16_t *latent, const int64_t *slots, int64_t n, int8_t *cache,
                      int64_t n_rows)
{
    for (int64_t i = 0; i < n; i++) {
        int64_t slot = slots[i];
        if (slot < 0) continue;
        if (slot >= n_rows) return -1;
        const uint16_t *x = latent + i * ORACLE_LATENT;
        double amax = 0.0;
        for (int j = 0; j < ORACLE_LATENT; j++) {
            double a = fabs(bf16(x[j]));
            if (a > amax) amax = a;
        }
        if (amax < amax_floor()) amax = amax_floor();
        float scale = (float)(amax / ORACLE_QMAX);
        unsigned char *row = (unsigned char *)cache + slot * ORACLE_ROW_BYTES;
        for (int j = 0; j < ORACLE_LATENT; j++) {
            double r = (double)(float)(bf16(x[j]) / (double)scale); /* fp32 quotient        */
            double c = nearbyint(r);                                /* ties to even         */
            if (c > ORACLE_QMAX) c = ORACLE_QMAX;
            if (c < -ORACLE_QMAX) c = -ORACLE_QMAX;
            row[j] = (unsigned char)(int8_t)c;
        }
        memcpy(row + ORACLE_LATENT, &scale, 4);
        memset(row + ORACLE_LATENT + 4, 0, ORACLE_ROW_BYTES - ORACLE_LATENT - 4);
    }
    return 0;
}

/* Dequantise one cache row into fp64 (code * scale). */
void oracle_dequant_row(const int8_t *cache, int64_t row, double *out)
{
    const unsigned char *r = (const unsigned char *)cache + row * ORACLE_ROW_BYTES;
    float scale;
    memcpy(&scale, r + ORACLE_LATENT, 4);
    for (int j = 0; j < ORACLE_LATENT; j++) out[j] = (double)(int8_t)r[j] * (double)scale;
}

/* ---------------------------------------------------------------------------------------------
 * layer_norm -- [DSA-REF] "layer_norm: nn.LayerNorm over the trailing d: mean-subtract,
 * variance-normalise, then w * x + b"; trap 1: k_norm is a LayerNorm with a bias.
 * Variance is the biased mean of squared deviations (the LayerNorm definition).
 * ------------------------------------------------------------------------------------------- */
void oracle_layer_norm(const double *x, int d, const double *w, const double *b, double eps,
                       double *y)
{
    double mean = 0.0;
    for (int i = 0; i < d; i++) mean += x[i];
    mean /= d;
    double var = 0.0;
    for (int i = 0; i < d; i++) var += (x[i] - mean) * (x[i] - mean);
    var /= d;
    double inv = 1.0 / sqrt(var + eps);
    for (int i = 0; i < d; i++) y[i] = (x[i] - mean) * inv * w[i] + b[i];
}

/* ---------------------------------------------------------------------------------------------
 * visible -- [DSA-REF] "visible: which keys a query at q_pos may see: causal and not padding".
 * A sequence occupies padded positions [0, pad + len); positions below pad are padding.
 * ------------------------------------------------------------------------------------------- */
int oracle_visible(int64_t pad, int64_t len, int64_t q_pos, int64_t t)
{
    return t >= pad && t <= q_pos && t < pad + len;
}

/* A pool exists only if all kpool slots are valid tokens ([DSA-REF] trap 4); pools start at the
 * first valid token ([DSA-REF] trap 3). */
int64_t oracle_n_pools(int64_t len, int kpool)
{
    return len / kpool;
}

/* The pools a query may use: existing pools whose every slot is visible (READING: a causal query
 * sees a pool only once all of its slots are visible; its visible remainder is the tail). Checked
 * pool by pool with `visible`, literally. */
int64_t oracle_n_visible_pools(int64_t pad, int64_t len, int64_t q_pos, int kpool)
{
    int64_t n = 0;
    for (int64_t p = 0; p < oracle_n_pools(len, kpool); p++) {
        int all = 1;
        for (int s = 0; s < kpool; s++) all &= oracle_visible(pad, len, q_pos, pad + p * kpool + s);
        if (!all) break;
        n++;
    }
    return n;
}

/* ---------------------------------------------------------------------------------------------
 * pool_states -- [DSA-REF] "pool_states: build the pools; k/gate are [seq, index_head_dim]",
 * trap 1 (k_norm LayerNorm with bias), trap 2 (softmax over the pool-slot axis, per channel),
 * trap 3 (pools start at the first valid token), trap 4 (only complete pools exist).
 *   pooled[p][d] = sum_s softmax_s(gate[t_s][d]) * LN(k[t_s])[d],  t_s = pad + kpool*p + s.
 * READINGS: gate is a separate per-token input, not normalised; k and gate rows are this
 * sequence's rows in padded coordinates (row t at k + t*d).
 * Returns the number of pools written.
 * ------------------------------------------------------------------------------------------- */
int64_t oracle_pool_states(const uint16_t *k, const uint16_t *gate, int d, int64_t pad,
                           int64_t len, int kpool, const float *ln_w, const float *ln_b,
                           double eps, double *pooled)
{
    double *w = malloc(sizeof(double) * d), *b = malloc(sizeof(double) * d);
    double *x = malloc(sizeof(double) * d);
    double *y = malloc(sizeof(double) * (size_t)d * kpool);
    double *g = malloc(sizeof(double) * kpool);
    for (int i = 0; i < d; i++) { w[i] = ln_w[i]; b[i] = ln_b[i]; }
    int64_t np_ = oracle_n_pools(len, kpool);
    for (int64_t p = 0; p < np_; p++) {
        for (int s = 0; s < kpool; s++) {
            int64_t t = pad + p * kpool + s;
            for (int i = 0; i < d; i++) x[i] = bf16(k[t * d + i]);
            oracle_layer_norm(x, d, w, b, eps, y + (size_t)s * d);
        }
        for (int i = 0; i < d; i++) {
            double m = -INFINITY;
            for (int s = 0; s < kpool; s++) {
                g[s] = bf16(gate[(pad + p * kpool + s) * d + i]);
                if (g[s] > m) m = g[s];
            }
            double den = 0.0, num = 0.0;
            for (int s = 0; s < kpool; s++) {
                double e = exp(g[s] - m);
                den += e;
                num += e * y[(size_t)s * d + i];
            }
            pooled[p * d + i] = num / den;
        }
    }
    free(w); free(b); free(x); free(y); free(g);
    return np_;
}

/* ---------------------------------------------------------------------------------------------
 * index_scores -- [DSA-REF] "index_scores: per-(query, pool) index score; the matmul -> relu ->
 * head-weighted sum chain"; [PYPTO] indexer 32 heads x 128.
 *   score[p] = sum_h w[h] * max(0, sum_d q[h][d] * pooled[p][d]),  p < n_vis.
 * READING: no further scale (any positive constant folds into w and leaves the top-k unchanged).
 * ------------------------------------------------------------------------------------------- */
void oracle_index_scores(const uint16_t *q_idx, const float *w, const double *pooled, int H,
                         int D, int64_t n_vis, double *scores)
{
    for (int64_t p = 0; p < n_vis; p++) {
        double s = 0.0;
        for (int h = 0; h < H; h++) {
            double dot = 0.0;
            for (int d = 0; d < D; d++) dot += bf16(q_idx[h * D + d]) * pooled[p * D + d];
            s += (double)w[h] * (dot > 0.0 ? dot : 0.0);
        }
        scores[p] = s;
    }
}

/* ---------------------------------------------------------------------------------------------
 * pool_q8 -- the INT8 indexer state: [PYPTO] "What is quantized" gives the indexer state cache as
 * FP32 and names the sibling port's INT8 form with one FP32 scale per row.
 * READING: a row is one pool's fp32 key (d values). It is quantized with the recipe of the latent
 * cache rows ([KERNELS] store_int8 and [PYPTO] "What is quantized"): amax floored at
 * INT8_AMAX_EPS, scale = fl32(amax / 127), code = clamp(round_half_even(fl32(x / scale)), +-127).
 * ------------------------------------------------------------------------------------------- */
void oracle_pool_q8(const float *x, int d, int8_t *codes, float *scale_out)
{
    double amax = 0.0;
    for (int j = 0; j < d; j++) {
        double a = fabs((double)x[j]);
        if (a > amax) amax = a;
    }
    if (amax < amax_floor()) amax = amax_floor();
    const float scale = (float)(amax / ORACLE_QMAX);
    for (int j = 0; j < d; j++) {
        double r = (double)(float)((double)x[j] / (double)scale); /* fp32 quotient        */
        double c = nearbyint(r);                                  /* ties to even         */
        if (c > ORACLE_QMAX) c = ORACLE_QMAX;
        if (c < -ORACLE_QMAX) c = -ORACLE_QMAX;
        codes[j] = (int8_t)c;
    }
    *scale_out = scale;
}

/* ---------------------------------------------------------------------------------------------
 * index_scores on the INT8 indexer state: the index_scores chain with each pooled key replaced by
 * its dequantised value code * scale:
 *   score[p] = sum_h w[h] * max(0, sum_d q[h][d] * codes[p][d] * scale[p]),  p < n_vis.
 * ------------------------------------------------------------------------------------------- */
void oracle_index_scores_q8(const uint16_t *q_idx, const float *w, const int8_t *codes,
                            const float *scales, int H, int D, int64_t n_vis, double *scores)
{
    for (int64_t p = 0; p < n_vis; p++) {
        double s = 0.0;
        for (int h = 0; h < H; h++) {
            double dot = 0.0;
            for (int d = 0; d < D; d++)
                dot += bf16(q_idx[h * D + d]) * ((double)codes[p * D + d] * (double)scales[p]);
            s += (double)w[h] * (dot > 0.0 ? dot : 0.0);
        }
        scores[p] = s;
    }
}

/* ---------------------------------------------------------------------------------------------
 * topk_pools -- [DSA-REF] "topk_pools: select up to select_k pools per query".
 * READINGS: the order is score descending, ties to the lower pool id (-0.0 equals +0.0); fewer
 * than select_k visible pools selects them all; the rest of the row is INVALID.
 * Returns n_sel = min(select_k, n_vis).
 * ------------------------------------------------------------------------------------------- */
static const double *g_sort_scores;
static int by_score_then_id(const void *a, const void *b)
{
    int32_t i = *(const int32_t *)a, j = *(const int32_t *)b;
    double si = g_sort_scores[i], sj = g_sort_scores[j];
    if (si > sj) return -1;
    if (si < sj) return 1;
    return (i > j) - (i < j);
}

int64_t oracle_topk_pools(const double *scores, int64_t n_vis, int64_t select_k, int32_t *out)
{
    int32_t *ids = malloc(sizeof(int32_t) * (n_vis > 0 ? n_vis : 1));
    for (int64_t p = 0; p < n_vis; p++) ids[p] = (int32_t)p;
    g_sort_scores = scores;
    qsort(ids, (size_t)n_vis, sizeof(int32_t), by_score_then_id);
    int64_t n_sel = n_vis < select_k ? n_vis : select_k;
    for (int64_t i = 0; i < select_k; i++) out[i] = i < n_sel ? ids[i] : ORACLE_INVALID;
    free(ids);
    return n_sel;
}

/* ---------------------------------------------------------------------------------------------
 * expand_selection -- [DSA-REF] "expand_selection: expand selected pools into raw token indices,
 * append the visible tail, pad with INVALID"; trap 6: all out_width entries are written.
 * Pool p covers tokens pad + kpool*p + s, s ascending (trap 3). The tail is every visible token
 * after the last visible pool, ascending (trap 4: a partial pool is handled by the tail).
 * READING: pools appear in the order topk_pools returns them.
 * Returns the number of valid entries, or -1 if they do not fit in out_width.
 * ------------------------------------------------------------------------------------------- */
int64_t oracle_expand_selection(const int32_t *topk, int64_t n_sel, int64_t pad, int64_t len,
                                int64_t q_pos, int kpool, int64_t out_width, int32_t *tok_out)
{
    int64_t n_vis = oracle_n_visible_pools(pad, len, q_pos, kpool);
    int64_t j = 0;
    for (int64_t i = 0; i < out_width; i++) tok_out[i] = ORACLE_INVALID;
    for (int64_t i = 0; i < n_sel; i++) {
        for (int s = 0; s < kpool; s++) {
            if (j >= out_width) return -1;
            tok_out[j++] = (int32_t)(pad + (int64_t)topk[i] * kpool + s);
        }
    }
    for (int64_t t = pad + n_vis * kpool; oracle_visible(pad, len, q_pos, t); t++) {
        if (j >= out_width) return -1;
        tok_out[j++] = (int32_t)t;
    }
    return j;
}

/* Map token positions of one sequence to cache rows through its slot map; INVALID stays. */
void oracle_rows_from_tokens(const int32_t *tok, int64_t width, const int64_t *slot_map_row,
                             int32_t *rows_out)
{
    for (int64_t i = 0; i < width; i++)
        rows_out[i] = tok[i] < 0 ? ORACLE_INVALID : (int32_t)slot_map_row[tok[i]];
}

/* ---------------------------------------------------------------------------------------------
 * sparse NoPE MLA over gathered int8 rows -- [KERNELS] "titan_mla.triton_mla_sparse_attention":
 * int8 dequantisation, the shared 512-d latent used as both K and V, fp32 softmax and
 * accumulation (here fp64); "The tested MLA contract": one KV head, negative index padding;
 * [DSA-REF] "mla_masked_attention: NoPE MLA over a per-query selected key set".
 *   c_j = code_j * scale_j;  s_hj = sm_scale * q_h . c_j;  o_h = sum_j softmax_j(s_h)_j c_j;
 *   lse_h = max_j s_hj + log(sum_j exp(s_hj - max)).
 * Each non-negative index entry is one key. READING: no valid entry gives o = 0, lse = -inf.
 * Returns 0, or -1 if an index is past the cache (outside the contract).
 * ------------------------------------------------------------------------------------------- */
int oracle_sparse_mla(const uint16_t *q, int Hm, const int8_t *cache, int64_t n_rows,
                      const int32_t *rows, int64_t width, double sm_scale, double *out, double *lse)
{
    const int L = ORACLE_LATENT;
    int64_t nv = 0;
    for (int64_t j = 0; j < width; j++) {
        if (rows[j] >= n_rows) return -1;
        if (rows[j] >= 0) nv++;
    }
    double *c = malloc(sizeof(double) * (size_t)(nv > 0 ? nv : 1) * L);
    double *s = malloc(sizeof(double) * (size_t)(nv > 0 ? nv : 1));
    int64_t v = 0;
    for (int64_t j = 0; j < width; j++)
        if (rows[j] >= 0) oracle_dequant_row(cache, rows[j], c + (size_t)(v++) * L);
    for (int h = 0; h < Hm; h++) {
        double *o = out + (size_t)h * L;
        for (int d = 0; d < L; d++) o[d] = 0.0;
        if (nv == 0) { lse[h] = -INFINITY; continue; }
        double m = -INFINITY;
        for (int64_t j = 0; j < nv; j++) {
            double dot = 0.0;
            for (int d = 0; d < L; d++) dot += bf16(q[(size_t)h * L + d]) * c[(size_t)j * L + d];
            s[j] = sm_scale * dot;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < nv; j++) {
            double p = exp(s[j] - m);
            l += p;
            for (int d = 0; d < L; d++) o[d] += p * c[(size_t)j * L + d];
        }
        for (int d = 0; d < L; d++) o[d] /= l;
        lse[h] = m + log(l);
    }
    free(c); free(s);
    return 0;
}

/* ---------------------------------------------------------------------------------------------
 * topk_to_mask -- [DSA-REF] "topk_to_mask: turn an index row into the boolean visibility mask
 * the attention consumes". Entries are token positions in [0, n_tok); INVALID is skipped.
 * ------------------------------------------------------------------------------------------- */
void oracle_topk_to_mask(const int32_t *tok, int64_t width, int64_t n_tok, uint8_t *mask)
{
    memset(mask, 0, (size_t)n_tok);
    for (int64_t i = 0; i < width; i++)
        if (tok[i] >= 0 && tok[i] < n_tok) mask[tok[i]] = 1;
}

/* Dense masked form of the same attention ([DSA-REF] mla_masked_attention over a boolean mask):
 * every position t of the sequence with mask[t] set and a cache row contributes once. Used as an
 * independent cross-check of the gather form on inputs without duplicate indices. */
int oracle_masked_attention(const uint16_t *q, int Hm, const int8_t *cache, int64_t n_rows,
                            const int64_t *slot_map_row, int64_t n_tok, const uint8_t *mask,
                            double sm_scale, double *out, double *lse)
{
    const int L = ORACLE_LATENT;
    double *c = malloc(sizeof(double) * L);
    double *m = malloc(sizeof(double) * Hm), *l = malloc(sizeof(double) * Hm);
    for (int h = 0; h < Hm; h++) { m[h] = -INFINITY; l[h] = 0.0; }
    for (int64_t i = 0; i < (int64_t)Hm * L; i++) out[i] = 0.0;
    /* two passes: maxima, then exp-weighted sums (no online rescaling, so the order of terms
     * differs from the gather form only in which rows come first) */
    for (int pass = 0; pass < 2; pass++) {
        for (int64_t t = 0; t < n_tok; t++) {
            if (!mask[t] || slot_map_row[t] < 0) continue;
            if (slot_map_row[t] >= n_rows) { free(c); free(m); free(l); return -1; }
            oracle_dequant_row(cache, slot_map_row[t], c);
            for (int h = 0; h < Hm; h++) {
                double dot = 0.0;
                for (int d = 0; d < L; d++) dot += bf16(q[(size_t)h * L + d]) * c[d];
                double s = sm_scale * dot;
                if (pass == 0) {
                    if (s > m[h]) m[h] = s;
                } else {
                    double p = exp(s - m[h]);
                    l[h] += p;
                    for (int d = 0; d < L; d++) out[(size_t)h * L + d] += p * c[d];
                }
            }
        }
    }
    for (int h = 0; h < Hm; h++) {
        if (l[h] == 0.0) { lse[h] = -INFINITY; continue; }
        for (int d = 0; d < L; d++) out[(size_t)h * L + d] /= l[h];
        lse[h] = m[h] + log(l[h]);
    }
    free(c); free(m); free(l);
    return 0;
}

/* =============================================================================================
 * The MLA up-projection (the step after the sparse attention; NEXT-3 of the build)
 * [DSA-REF] "expand_kv: expand the compressed latent into per-head K and V", with kv_b_proj in
 * the "linear: y = x @ w^T" layout (w is [out, in]); [GLM-5.3-Flash] 'Checkpoint shape':
 * 64 heads, kv_lora_rank 512, qk_head_dim = v_head_dim = 256, qk_rope_head_dim 0.
 * READING: the rows of kv_b_proj are grouped per head, the dk K rows of head h first, then its
 * dv V rows: row h (dk + dv) + e. The weights are bf16 (the checkpoint's kv_b_proj dtype,
 * [GLM-5.3-Flash] 'Open questions': "kv_b_proj is BF16 in the checkpoint").
 * The absorbed form that the sparse MLA computes in latent space meets the expanded form through
 *   q_h . K_h,t = (q_h W_k,h) . c_t        and        sum_t p_t V_h,t = (sum_t p_t c_t) W_v,h^T.
 * ============================================================================================= */

/* K[h][t][e] = sum_d c[t][d] W[h (dk+dv) + e][d];  V[h][t][e] = sum_d c[t][d] W[h (dk+dv) + dk + e][d].
 * c is [T][L]; K is [Hm][T][dk], V is [Hm][T][dv]. */
void oracle_expand_kv(const double *c, int64_t T, int L, const uint16_t *w, int Hm, int dk, int dv,
                      double *k_out, double *v_out)
{
    for (int h = 0; h < Hm; h++) {
        const uint16_t *wh = w + (size_t)h * (dk + dv) * L;
        for (int64_t t = 0; t < T; t++) {
            for (int e = 0; e < dk + dv; e++) {
                double s = 0.0;
                for (int d = 0; d < L; d++) s += c[(size_t)t * L + d] * bf16(wh[(size_t)e * L + d]);
                if (e < dk) k_out[((size_t)h * T + t) * dk + e] = s;
                else v_out[((size_t)h * T + t) * dv + (e - dk)] = s;
            }
        }
    }
}

/* The latent-space query of the absorbed form: q_lat[h][d] = sum_e q[h][e] W[h (dk+dv) + e][d]
 * for the dk K rows of head h (q is [Hm][dk], q_lat is [Hm][L]). */
void oracle_q_absorb(const double *q, int Hm, int L, const uint16_t *w, int dk, int dv, double *q_lat)
{
    for (int h = 0; h < Hm; h++) {
        const uint16_t *wh = w + (size_t)h * (dk + dv) * L;
        for (int d = 0; d < L; d++) {
            double s = 0.0;
            for (int e = 0; e < dk; e++) s += q[(size_t)h * dk + e] * bf16(wh[(size_t)e * L + d]);
            q_lat[(size_t)h * L + d] = s;
        }
    }
}

/* The up-projection epilogue of the absorbed form: out[h][e] = sum_d o_lat[h][d] W[h (dk+dv) + dk + e][d]
 * for the dv V rows of head h (o_lat is [Hm][L], out is [Hm][dv]). */
void oracle_v_up(const double *o_lat, int Hm, int L, const uint16_t *w, int dk, int dv, double *out)
{
    for (int h = 0; h < Hm; h++) {
        const uint16_t *wv = w + ((size_t)h * (dk + dv) + dk) * L;
        for (int e = 0; e < dv; e++) {
            double s = 0.0;
            for (int d = 0; d < L; d++) s += o_lat[(size_t)h * L + d] * bf16(wv[(size_t)e * L + d]);
            out[(size_t)h * dv + e] = s;
        }
    }
}

/* Softmax attention of Hm queries over T keys in fp64 (the definition, max-subtracted):
 *   out[h] = sum_t softmax_t(scale * q[h] . K[t]) V[t],
 * with K, V per head ([Hm][T][dq] and [Hm][T][dvv]) when shared == 0, or one set for every head
 * ([T][dq], [T][dvv]) when shared != 0 (the latent form: K = V = the latent rows). */
void oracle_attention_f64(const double *q, int Hm, int dq, const double *k, const double *v, int64_t T,
                          int dvv, int shared, double scale, double *out)
{
    double *s = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    for (int h = 0; h < Hm; h++) {
        const double *kh = shared ? k : k + (size_t)h * T * dq;
        const double *vh = shared ? v : v + (size_t)h * T * dvv;
        double *o = out + (size_t)h * dvv;
        for (int e = 0; e < dvv; e++) o[e] = 0.0;
        if (T == 0) continue;
        double m = -INFINITY;
        for (int64_t t = 0; t < T; t++) {
            double dot = 0.0;
            for (int d = 0; d < dq; d++) dot += q[(size_t)h * dq + d] * kh[(size_t)t * dq + d];
            s[t] = scale * dot;
            if (s[t] > m) m = s[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < T; t++) {
            const double p = exp(s[t] - m);
            l += p;
            for (int e = 0; e < dvv; e++) o[e] += p * vh[(size_t)t * dvv + e];
        }
        for (int e = 0; e < dvv; e++) o[e] /= l;
    }
    free(s);
}

/* =============================================================================================
 * The FP8 latent cache row (NEXT-4 of the build). [GLM on CUDA] names an opt-in "FP8 or 4-bit
 * latent cache (--kv-dtype fp8 / fp4), lossy" and gives no format.
 * READINGS: FP8 is E4M3 in its OCP "E4M3FN" form (exponent bias 7, subnormals, no infinities,
 * S.1111.111 is NaN, largest finite value 448); the row is the INT8 row's layout and recipe with
 * 448 in place of 127: scale = fl32(max(amax, floor) / 448), code = the E4M3 value nearest
 * fl32(x / scale) with ties to the even code (even mantissa), saturating at +-448, the sign kept
 * (-0 gives 0x80); bytes: 512 codes, the fp32 scale (little endian), 12 zero bytes. The
 * dequantised value is value(code) * scale.
 * ============================================================================================= */
#define ORACLE_E4M3_MAX 448.0

/* The value of an E4M3 code: (1 + m/8) 2^(e-7) for exponent field e >= 1, (m/8) 2^-6 for e = 0. */
double oracle_e4m3_value(unsigned code)
{
    const int s = (int)((code >> 7) & 1u), e = (int)((code >> 3) & 15u), m = (int)(code & 7u);
    if (e == 15 && m == 7) return NAN;
    const double v = e == 0 ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
    return s ? -v : v;
}

/* The E4M3 code nearest x (ties to the even code), saturating at +-448. */
unsigned oracle_e4m3_encode(double x)
{
    if (x != x) return 0x7Fu;
    const unsigned s = signbit(x) ? 0x80u : 0u;
    const double a = fabs(x);
    if (a >= ORACLE_E4M3_MAX) return s | 0x7Eu;
    unsigned code;
    if (a < ldexp(1.0, -6)) {                     /* subnormal range: steps of 2^-9; 8 is 2^-6 */
        code = (unsigned)nearbyint(ldexp(a, 9));
    } else {
        int e;
        frexp(a, &e);                             /* a in [2^(e-1), 2^e)                      */
        const int E = e - 1;
        unsigned m = (unsigned)nearbyint(ldexp(a, 3 - E));   /* in [8, 16]                    */
        int field = E + 7;
        if (m == 16u) { m = 8u; field++; }
        code = ((unsigned)field << 3) | (m - 8u);
        if (code > 0x7Eu) code = 0x7Eu;
    }
    return s | code;
}

/* store of FP8 rows: the store_int8 contract with E4M3 codes. Returns 0, or -1 if a slot is past
 * the cache. */
int oracle_store_fp8(const uint16_t *latent, const int64_t *slots, int64_t n, uint8_t *cache, int64_t n_rows)
{
    for (int64_t i = 0; i < n; i++) {
        const int64_t slot = slots[i];
        if (slot < 0) continue;
        if (slot >= n_rows) return -1;
        const uint16_t *x = latent + i * ORACLE_LATENT;
        double amax = 0.0;
        for (int j = 0; j < ORACLE_LATENT; j++) {
            const double a = fabs(bf16(x[j]));
            if (a > amax) amax = a;
        }
        if (amax < amax_floor()) amax = amax_floor();
        const float scale = (float)(amax / ORACLE_E4M3_MAX);
        unsigned char *row = cache + slot * ORACLE_ROW_BYTES;
        for (int j = 0; j < ORACLE_LATENT; j++)
            row[j] = (unsigned char)oracle_e4m3_encode((double)(float)(bf16(x[j]) / (double)scale));
        memcpy(row + ORACLE_LATENT, &scale, 4);
        memset(row + ORACLE_LATENT + 4, 0, ORACLE_ROW_BYTES - ORACLE_LATENT - 4);
    }
    return 0;
}

/* Dequantise one FP8 cache row into fp64 (value(code) * scale). */
void oracle_dequant_row_fp8(const uint8_t *cache, int64_t row, double *out)
{
    const unsigned char *r = cache + row * ORACLE_ROW_BYTES;
    float scale;
    memcpy(&scale, r + ORACLE_LATENT, 4);
    for (int j = 0; j < ORACLE_LATENT; j++) out[j] = oracle_e4m3_value(r[j]) * (double)scale;
}

/* =============================================================================================
 * The 4-bit latent cache row (NEXT-4 of the build). [GLM on CUDA] names the opt-in "--kv-dtype
 * fp4" latent cache and gives no layout.
 * READINGS: FP4 is E2M1 (sign bit, two exponent bits with bias 1, one mantissa bit: magnitudes
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6) with two levels of scale, one E4M3 scale for every 16 consecutive
 * values and one fp32 scale for the row (the block-scaled FP4 form of the sm_100 tensor cores):
 *   s_row = fl32(max(amax, floor) / 2688)     2688 = 6 * 448, the largest code times the
 *                                             largest block scale
 *   e_k   = the E4M3 code nearest fl32(bmax_k / fl32(6 s_row)) (bmax_k the largest |x| of block
 *           k; ties to the even code, saturating at 448)
 *   d_k   = fl32(value(e_k) s_row)
 *   code  = the E2M1 code nearest fl32(x / d_k), ties to the even code, saturating at +-6, the
 *           sign kept; 0 where d_k = 0
 * bytes: [0, 256) code pairs (byte i holds dim 2i in its low nibble and dim 2i + 1 in its high
 * one), [256, 288) the 32 block scales, [288, 292) s_row (little endian), [292, 304) zeros. The
 * dequantised value is value(code) value(e_k) s_row.
 * ============================================================================================= */
#define ORACLE_FP4_ROW_BYTES 304
#define ORACLE_FP4_BLOCK 16
#define ORACLE_FP4_SCALES_AT 256
#define ORACLE_FP4_ROW_SCALE_AT 288
#define ORACLE_E2M1_MAX 6.0

/* The value of an E2M1 code: (1 + m/2) 2^(e-1) for exponent field e >= 1, m/2 for e = 0. */
double oracle_e2m1_value(unsigned code)
{
    const int s = (int)((code >> 3) & 1u), e = (int)((code >> 1) & 3u), m = (int)(code & 1u);
    const double v = e == 0 ? 0.5 * m : ldexp(2.0 + m, e - 2);
    return s ? -v : v;
}

/* The E2M1 code nearest x (ties to the even code), saturating at +-6, the sign kept. */
unsigned oracle_e2m1_encode(double x)
{
    const unsigned s = signbit(x) ? 8u : 0u;
    const double a = fabs(x);
    if (a >= ORACLE_E2M1_MAX) return s | 7u;
    unsigned code;
    if (a < 1.0) {                                /* subnormal range: steps of 0.5; 2 is 1.0   */
        code = (unsigned)nearbyint(2.0 * a);
    } else {
        int e;
        frexp(a, &e);                             /* a in [2^(e-1), 2^e)                      */
        const int E = e - 1;
        unsigned m = (unsigned)nearbyint(ldexp(a, 1 - E));   /* in [2, 4]                     */
        int field = E + 1;
        if (m == 4u) { m = 2u; field++; }
        code = ((unsigned)field << 1) | (m - 2u);
        if (code > 7u) code = 7u;
    }
    return s | code;
}

/* store of 4-bit rows (uint8 [n_rows, 304]). Returns 0, or -1 if a slot is past the cache. */
int oracle_store_fp4(const uint16_t *latent, const int64_t *slots, int64_t n, uint8_t *cache, int64_t n_rows)
{
    for (int64_t i = 0; i < n; i++) {
        const int64_t slot = slots[i];
        if (slot < 0) continue;
        if (slot >= n_rows) return -1;
        const uint16_t *x = latent + i * ORACLE_LATENT;
        double amax = 0.0;
        for (int j = 0; j < ORACLE_LATENT; j++) {
            const double a = fabs(bf16(x[j]));
            if (a > amax) amax = a;
        }
        if (amax < amax_floor()) amax = amax_floor();
        const float s_row = (float)(amax / (6.0 * ORACLE_E4M3_MAX));
        const float u = (float)(6.0 * (double)s_row);
        unsigned char *row = cache + slot * ORACLE_FP4_ROW_BYTES;
        memset(row, 0, ORACLE_FP4_ROW_BYTES);
        for (int k = 0; k < ORACLE_LATENT / ORACLE_FP4_BLOCK; k++) {
            const uint16_t *xb = x + k * ORACLE_FP4_BLOCK;
            double bmax = 0.0;
            for (int j = 0; j < ORACLE_FP4_BLOCK; j++) {
                const double a = fabs(bf16(xb[j]));
                if (a > bmax) bmax = a;
            }
            const unsigned e = oracle_e4m3_encode((double)(float)(bmax / (double)u));
            const float d = (float)(oracle_e4m3_value(e) * (double)s_row);
            row[ORACLE_FP4_SCALES_AT + k] = (unsigned char)e;
            for (int j = 0; j < ORACLE_FP4_BLOCK; j++) {
                const unsigned c = d > 0.0f ? oracle_e2m1_encode((double)(float)(bf16(xb[j]) / (double)d)) : 0u;
                const int dim = k * ORACLE_FP4_BLOCK + j;
                row[dim / 2] |= (unsigned char)((dim & 1) ? c << 4 : c);
            }
        }
        memcpy(row + ORACLE_FP4_ROW_SCALE_AT, &s_row, 4);
    }
    return 0;
}

/* Dequantise one 4-bit cache row into fp64 (value(code) value(e_k) s_row). */
void oracle_dequant_row_fp4(const uint8_t *cache, int64_t row, double *out)
{
    const unsigned char *r = cache + row * ORACLE_FP4_ROW_BYTES;
    float s_row;
    memcpy(&s_row, r + ORACLE_FP4_ROW_SCALE_AT, 4);
    for (int j = 0; j < ORACLE_LATENT; j++) {
        const unsigned c = (j & 1) ? (r[j / 2] >> 4) & 15u : r[j / 2] & 15u;
        const unsigned e = r[ORACLE_FP4_SCALES_AT + j / ORACLE_FP4_BLOCK];
        out[j] = oracle_e2m1_value(c) * oracle_e4m3_value(e) * (double)s_row;
    }
}
