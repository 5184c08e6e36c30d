// api.cu -- the C ABI (include/glm_dsa.h): host-side argument checks, workspace sizing and the
// kernel launches of each entry point. Nothing is enqueued unless every check passes.
#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"
#include "select.cuh"

namespace {
thread_local int g_last_cuda_error = 0;
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

namespace glm {
namespace abi {

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return GLM_OK;
    g_last_cuda_error = static_cast<int>(e);
    return GLM_ERR_CUDA;
}

int num_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

int check_mla(const glm_dsa_dims *dims, const void *q, const int8_t *cache, int64_t n_rows, const int32_t *rows,
              int32_t n_q, int32_t width, float sm_scale, const void *out, const float *lse, const float *out_f32) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_q < 0 || n_rows < 0 || width < 1 || width > 65536 || n_q > 65535) return GLM_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale)) return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (!q || !rows || !out || (n_rows > 0 && !cache)) return GLM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || (cache && !aligned(cache, 16)) || !aligned(rows, 4) || !aligned(out, 16) ||
        (lse && !aligned(lse, 4)) || (out_f32 && !aligned(out_f32, 16)))
        return GLM_ERR_INVALID_ARG;
    return GLM_OK;
}

}  // namespace abi
}  // namespace glm

namespace {
using glm::abi::check_mla;
using glm::abi::cuda_status;
using glm::abi::num_sms;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace of a selection (first in the workspace of both selection entry points): per query
// two 2048-bin histograms of score keys and kCntWords counters (zeroed by one kernel before a
// selection that spans several CTAs), the sample keys the CTAs of the fused index kernel publish
// (kSampleUnion per query; the selection on given scores uses none), the list sizes of each
// CTA, and the per-CTA regions of list A (candidates above the boundary bin) and list B (the
// boundary bin).
struct SelWs {
    unsigned *hist;
    unsigned *hist2;
    unsigned *counters;
    unsigned *fine;
    unsigned *words;
    unsigned long long *alist;
    unsigned long long *blist;
    size_t zero_bytes;   // hist, hist2 and counters
};
size_t sel_zero_bytes(int n_q) {
    return static_cast<size_t>(n_q) * (2 * glm::kHistBins + glm::kCntWords) * sizeof(unsigned);
}
size_t sel_fine_bytes(int n_q) { return align_up(static_cast<size_t>(n_q) * glm::kSampleUnion * sizeof(unsigned), 256); }
size_t sel_list_bytes(int n_q, int64_t ld) {
    return align_up(static_cast<size_t>(n_q) * static_cast<size_t>(glm::sel_list_cap(ld)) *
                    sizeof(unsigned long long), 256);
}
size_t sel_words_bytes(int n_q) { return align_up(static_cast<size_t>(n_q) * glm::kMaxSelCtas * sizeof(unsigned), 256); }
size_t sel_bytes(int n_q, int64_t ld) {
    return align_up(sel_zero_bytes(n_q), 256) + sel_fine_bytes(n_q) + sel_words_bytes(n_q) + 2 * sel_list_bytes(n_q, ld);
}
// The score rows of the selection ([n_q][ld] fp32) and, for many queries, the scratch of the
// GEMM scoring path (queries as scaled fp16, w', visible counts), laid out after sel_bytes.
size_t score_rows_bytes(int n_q, int64_t ld) {
    return align_up(static_cast<size_t>(n_q) * static_cast<size_t>(ld > 0 ? ld : 0) * sizeof(float), 256);
}
size_t gemm_scratch_bytes(int n_q) {
    return n_q >= glm::kIndexGemmMinQueries ? align_up(glm::index_gemm_scratch_bytes(n_q), 256) : 0;
}
// fp32 keys, many queries: scores by the GEMM kernel, then the selection on them.
bool index_by_gemm(int n_q, int64_t ld_pools, int batch, bool int8_keys) {
    return !int8_keys && n_q >= glm::kIndexGemmMinQueries && ld_pools > 0 && batch <= 65535;
}
SelWs sel_layout(void *base, int n_q, int64_t ld) {
    char *p = static_cast<char *>(base);
    SelWs w;
    w.hist = reinterpret_cast<unsigned *>(p);
    w.hist2 = w.hist + static_cast<size_t>(n_q) * glm::kHistBins;
    w.counters = w.hist2 + static_cast<size_t>(n_q) * glm::kHistBins;
    w.zero_bytes = sel_zero_bytes(n_q);
    p += align_up(w.zero_bytes, 256);
    w.fine = reinterpret_cast<unsigned *>(p);
    p += sel_fine_bytes(n_q);
    w.words = reinterpret_cast<unsigned *>(p);
    p += sel_words_bytes(n_q);
    w.alist = reinterpret_cast<unsigned long long *>(p);
    p += sel_list_bytes(n_q, ld);
    w.blist = reinterpret_cast<unsigned long long *>(p);
    return w;
}

// Workspace of the sparse MLA: partial accumulators and (m, l) pairs per (query, part, head),
// then a 256-byte tail whose first word is the kernels' status (nonzero after a timed-out wait).
// Sized for the plan of n_q queries and for every smaller count: up to the few-query maximum
// the plan keeps one partial per chunk; above it at most that many partials, or one per query.
size_t mla_parts(int n_q, int n_heads, int width) {
    const int sms = num_sms();
    const long long chunks = (width + glm::mla_tc_chunk() - 1) / glm::mla_tc_chunk();
    const long long few_max = glm::mla_few_query_max(n_heads, sms);
    if (n_q <= few_max) return static_cast<size_t>(n_q) * static_cast<size_t>(chunks) * n_heads;
    const glm::MlaPlan p = glm::mla_plan(n_q, n_heads, width, sms);
    const long long per = static_cast<long long>(n_q) * p.n_parts;
    return static_cast<size_t>(per > few_max * chunks ? per : few_max * chunks) * n_heads;
}
size_t mla_acc_bytes(size_t parts) { return align_up(parts * glm::kLatent * sizeof(float), 256); }
size_t mla_ml_bytes(size_t parts) { return align_up(parts * 2 * sizeof(float), 256); }
// Host checks of each stage's arguments (GLM_OK: may proceed; a count of zero is accepted).
int check_store(const glm_dsa_dims *dims, const void *latent, const int64_t *slots, int64_t n,
                const int8_t *cache, int64_t n_rows) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n < 0 || n_rows < 0) return GLM_ERR_INVALID_ARG;
    if (n == 0) return GLM_OK;
    if (!latent || !slots || !cache) return GLM_ERR_INVALID_ARG;
    if (!aligned(latent, 16) || !aligned(cache, 16) || !aligned(slots, 8)) return GLM_ERR_INVALID_ARG;
    return GLM_OK;
}

int check_kpool(const glm_dsa_dims *dims, const void *k, const void *gate, int64_t ld_tokens,
                const float *ln_w, const float *ln_b, float ln_eps, const int32_t *pad, const int32_t *len,
                const int32_t *pool_begin, int32_t batch, int32_t max_new_pools, const void *pooled,
                int64_t ld_pools, const int32_t *n_pools) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (batch < 0 || max_new_pools < 0 || ld_tokens < 0 || ld_pools < 0) return GLM_ERR_INVALID_ARG;
    if (!(ln_eps >= 0.0f)) return GLM_ERR_INVALID_ARG;
    if (batch == 0) return GLM_OK;
    if (!k || !gate || !ln_w || !ln_b || !pad || !len || !pooled) return GLM_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(gate, 16) || !aligned(ln_w, 16) || !aligned(ln_b, 16) ||
        !aligned(pooled, 16) || !aligned(pad, 4) || !aligned(len, 4) ||
        (pool_begin && !aligned(pool_begin, 4)) || (n_pools && !aligned(n_pools, 4)))
        return GLM_ERR_INVALID_ARG;
    if (static_cast<int64_t>(batch) * max_new_pools > (int64_t(1) << 40)) return GLM_ERR_INVALID_ARG;
    return GLM_OK;
}

size_t mla_workspace(int n_q, int n_heads, int width) {
    const size_t parts = mla_parts(n_q, n_heads, width);
    return mla_acc_bytes(parts) + mla_ml_bytes(parts) + 256;
}

// Workspace of a fused step: the selection's (with its score rows), the attention's, and a
// 256-byte status tail shared by every kernel of the step.
struct StepLayout {
    size_t idx, mla, total;
};
StepLayout step_layout(const glm_dsa_dims *dims, int n_q, int64_t ld, int width) {
    StepLayout L;
    const size_t idx = sel_bytes(n_q, ld) + score_rows_bytes(n_q, ld) + gemm_scratch_bytes(n_q) + 256;
    L.idx = 0;
    L.mla = idx;
    L.total = idx + mla_workspace(n_q, dims->n_heads, width) + 256;
    return L;
}

}  // namespace

extern "C" {

int glm_check_dims(const glm_dsa_dims *d) {
    if (d == nullptr) return GLM_ERR_INVALID_ARG;
    if (d->qk_rope_head_dim != 0) return GLM_ERR_UNSUPPORTED;  // NoPE only: zero-width rope slice
    if (d->kv_lora_rank != glm::kLatent || d->index_n_heads != glm::kIdxHeads ||
        d->index_head_dim != glm::kIdxDim || d->index_kpool != glm::kKpool)
        return GLM_ERR_UNSUPPORTED;
    if (d->n_heads < 1 || d->n_heads > glm::kMaxHeads) return GLM_ERR_UNSUPPORTED;
    if (d->index_topk <= 0 || d->index_topk % d->index_kpool != 0) return GLM_ERR_INVALID_ARG;
    return GLM_OK;
}

const char *glm_status_string(int s) {
    switch (s) {
        case GLM_OK: return "ok";
        case GLM_ERR_INVALID_ARG: return "invalid argument";
        case GLM_ERR_UNSUPPORTED: return "unsupported geometry";
        case GLM_ERR_WORKSPACE: return "workspace missing or too small";
        case GLM_ERR_CUDA: return "CUDA launch failed";
        default: return "unknown status";
    }
}

int glm_last_cuda_error(void) { return g_last_cuda_error; }

int glm_debug_set_cross_cta_wait_limit(uint32_t polls) {
    return cuda_status(glm::set_cross_cta_wait_limit(polls));
}

int glm_kv_store_int8(const glm_dsa_dims *dims, const void *latent, const int64_t *slots,
                      int64_t n, int8_t *cache, int64_t n_rows, void *stream) {
    const int rc = check_store(dims, latent, slots, n, cache, n_rows);
    if (rc != GLM_OK || n == 0) return rc;
    return cuda_status(glm::launch_store_int8(latent, slots, n, cache, n_rows,
                                              static_cast<cudaStream_t>(stream), num_sms()));
}

int glm_kv_store_fp8(const glm_dsa_dims *dims, const void *latent, const int64_t *slots,
                     int64_t n, uint8_t *cache, int64_t n_rows, void *stream) {
    const int rc = check_store(dims, latent, slots, n, reinterpret_cast<int8_t *>(cache), n_rows);
    if (rc != GLM_OK || n == 0) return rc;
    return cuda_status(glm::launch_store_fp8(latent, slots, n, cache, n_rows,
                                             static_cast<cudaStream_t>(stream), num_sms()));
}

int glm_kv_store_fp4(const glm_dsa_dims *dims, const void *latent, const int64_t *slots,
                     int64_t n, uint8_t *cache, int64_t n_rows, void *stream) {
    const int rc = check_store(dims, latent, slots, n, reinterpret_cast<int8_t *>(cache), n_rows);
    if (rc != GLM_OK || n == 0) return rc;
    return cuda_status(glm::launch_store_fp4(latent, slots, n, cache, n_rows,
                                             static_cast<cudaStream_t>(stream), num_sms()));
}

int glm_kpool_build(const glm_dsa_dims *dims, const void *k, const void *gate, int64_t ld_tokens,
                    const float *ln_w, const float *ln_b, float ln_eps, const int32_t *pad,
                    const int32_t *len, const int32_t *pool_begin, int32_t batch,
                    int32_t max_new_pools, float *pooled, int64_t ld_pools, int32_t *n_pools,
                    void *stream) {
    const int rc = check_kpool(dims, k, gate, ld_tokens, ln_w, ln_b, ln_eps, pad, len, pool_begin, batch,
                               max_new_pools, pooled, ld_pools, n_pools);
    if (rc != GLM_OK || batch == 0) return rc;
    return cuda_status(glm::launch_kpool_build(k, gate, ld_tokens, ln_w, ln_b, ln_eps, pad, len,
                                               pool_begin, batch, max_new_pools, pooled, ld_pools,
                                               n_pools, static_cast<cudaStream_t>(stream), num_sms()));
}

int glm_kpool_build_q8(const glm_dsa_dims *dims, const void *k, const void *gate, int64_t ld_tokens,
                       const float *ln_w, const float *ln_b, float ln_eps, const int32_t *pad,
                       const int32_t *len, const int32_t *pool_begin, int32_t batch,
                       int32_t max_new_pools, int8_t *pooled_codes, float *pooled_scales, int64_t ld_pools,
                       int32_t *n_pools, void *stream) {
    const int rc = check_kpool(dims, k, gate, ld_tokens, ln_w, ln_b, ln_eps, pad, len, pool_begin, batch,
                               max_new_pools, pooled_codes, ld_pools, n_pools);
    if (rc != GLM_OK || batch == 0) return rc;
    if (!pooled_scales || !aligned(pooled_scales, 4)) return GLM_ERR_INVALID_ARG;
    return cuda_status(glm::launch_kpool_build(k, gate, ld_tokens, ln_w, ln_b, ln_eps, pad, len, pool_begin, batch,
                                               max_new_pools, nullptr, ld_pools, n_pools,
                                               static_cast<cudaStream_t>(stream), num_sms(), pooled_codes,
                                               pooled_scales));
}

int glm_dsa_step_plan(const glm_dsa_dims *dims, int32_t n_q, int64_t ld_pools, int32_t batch, int32_t width,
                      int32_t int8_keys, int32_t *launches, int32_t *paths) {
    const int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_q < 0 || ld_pools < 0 || batch < 0 || width < 1 || width > 65536 || !launches) return GLM_ERR_INVALID_ARG;
    int k = 1, f = 0;   // step_prep
    if (n_q > 0) {
        if (index_by_gemm(n_q, ld_pools, batch, int8_keys != 0)) {
            f |= GLM_PLAN_INDEX_MANY;
            k += 5;   // query preparation, scores, histogram, selection, expansion
        } else {
            k += 1;   // the fused scores + selection + expansion
        }
        const glm::MlaPlan plan = glm::mla_plan(n_q, dims->n_heads, width, num_sms());
        if (plan.multi) f |= GLM_PLAN_MLA_MANY;
        if (plan.combine) f |= GLM_PLAN_MLA_COMBINE;
        k += plan.combine ? 2 : 1;
    }
    *launches = k;
    if (paths) *paths = f;
    return GLM_OK;
}

size_t glm_dsa_workspace_size(const glm_dsa_dims *dims, int32_t op, int32_t n_q,
                              int64_t max_pools, int32_t select_k, int32_t width) {
    if (glm_check_dims(dims) != GLM_OK || n_q < 0) return static_cast<size_t>(-1);
    switch (op) {
        case GLM_OP_INDEX_SCORES_TOPK:
            if (max_pools < 0 || select_k < 1 || select_k > glm::kMaxSelect) return static_cast<size_t>(-1);
            return sel_bytes(n_q, max_pools) + score_rows_bytes(n_q, max_pools) + gemm_scratch_bytes(n_q) + 256;
        case GLM_OP_TOPK_POOLS:
            if (max_pools < 0 || select_k < 1 || select_k > glm::kMaxSelect) return static_cast<size_t>(-1);
            return sel_bytes(n_q, max_pools);
        case GLM_OP_SPARSE_MLA:
            if (width < 1 || width > 65536) return static_cast<size_t>(-1);
            return mla_workspace(n_q, dims->n_heads, width);
        case GLM_OP_DECODE_STEP:
            if (max_pools < 0 || select_k < 1 || select_k > glm::kMaxSelect || width < 1 || width > 65536)
                return static_cast<size_t>(-1);
            return step_layout(dims, n_q, max_pools, width).total;
        default:
            return static_cast<size_t>(-1);
    }
}

namespace {

int enqueue_index_select(const void *q_idx, const float *w, const void *keys, const float *key_scales,
                         int64_t ld_pools,
                         const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                         int32_t batch, int32_t n_q, int32_t select_k, const int64_t *slot_map, int64_t ld_slot,
                         int32_t out_width, float *scores, int32_t *topk, int32_t *n_sel, int32_t *tok,
                         int32_t *rows, void *workspace, int *status, bool zero, int sms, cudaStream_t st,
                         const int32_t *new_pool_begin = nullptr, int new_pools = -1);

// Checks shared by the two scoring + selection entry points; GLM_OK when the call may proceed.
int check_index_args(const glm_dsa_dims *dims, const void *q_idx, const float *w, const void *pooled,
                     int64_t ld_pools, const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad,
                     const int32_t *len, int32_t batch, int32_t n_q, int32_t select_k, const float *scores,
                     const int32_t *topk, const int32_t *n_sel) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_q < 0 || batch < 0 || ld_pools < 0 || select_k < 1 || select_k > glm::kMaxSelect ||
        n_q > 65535 || ld_pools > (int64_t(1) << 31) / 128)
        return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (batch == 0 || !q_idx || !w || !q_seq || !q_pos || !pad || !len || !topk) return GLM_ERR_INVALID_ARG;
    if (ld_pools > 0 && !pooled) return GLM_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(w, 4) || (pooled && !aligned(pooled, 16)) ||
        !aligned(q_seq, 4) || !aligned(q_pos, 4) || !aligned(pad, 4) || !aligned(len, 4) ||
        !aligned(topk, 4) || (n_sel && !aligned(n_sel, 4)) || (scores && !aligned(scores, 4)))
        return GLM_ERR_INVALID_ARG;
    return GLM_OK;
}

// Scores + selection (+ expansion when tok or rows is given) in one fused launch, preceded by
// the zeroing of the multi-CTA words when the selection spans several CTAs.
int run_index_select(const glm_dsa_dims *dims, const void *q_idx, const float *w, const void *pooled,
                     const float *key_scales,
                     int64_t ld_pools, const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad,
                     const int32_t *len, int32_t batch, int32_t n_q, int32_t select_k,
                     const int64_t *slot_map, int64_t ld_slot, int32_t out_width, float *scores,
                     int32_t *topk, int32_t *n_sel, int32_t *tok, int32_t *rows, void *workspace,
                     size_t ws_bytes, void *stream) {
    const size_t need = glm_dsa_workspace_size(dims, GLM_OP_INDEX_SCORES_TOPK, n_q, ld_pools, select_k, 0);
    if (workspace == nullptr || ws_bytes < need || !aligned(workspace, 256)) return GLM_ERR_WORKSPACE;
    int *status = reinterpret_cast<int *>(static_cast<char *>(workspace) + need - 256);
    return enqueue_index_select(q_idx, w, pooled, key_scales, ld_pools, q_seq, q_pos, pad, len, batch, n_q, select_k, slot_map,
                                ld_slot, out_width, scores, topk, n_sel, tok, rows, workspace, status, true,
                                num_sms(), static_cast<cudaStream_t>(stream));
}

}  // namespace

namespace {

// The fused index launch on a workspace laid out by sel_layout (+ the score rows); `zero`: also
// enqueue the zeroing of the multi-CTA words (false when the caller has zeroed them already).
int enqueue_index_select(const void *q_idx, const float *w, const void *keys, const float *key_scales,
                         int64_t ld_pools,
                         const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                         int32_t batch, int32_t n_q, int32_t select_k, const int64_t *slot_map, int64_t ld_slot,
                         int32_t out_width, float *scores, int32_t *topk, int32_t *n_sel, int32_t *tok,
                         int32_t *rows, void *workspace, int *status, bool zero, int sms, cudaStream_t st,
                         const int32_t *new_pool_begin, int new_pools) {
    const SelWs sw = sel_layout(workspace, n_q, ld_pools);
    char *ws = static_cast<char *>(workspace);
    float *sbuf = scores ? scores : reinterpret_cast<float *>(ws + sel_bytes(n_q, ld_pools));
    if (index_by_gemm(n_q, ld_pools, batch, key_scales != nullptr)) {
        // zero the selection's words, score every (query, pool), select, expand
        int rc = GLM_OK;
        if (zero) rc = cuda_status(glm::launch_zero(sw.hist, align_up(sw.zero_bytes, 16), st));
        if (rc != GLM_OK) return rc;
        void *scratch = ws + sel_bytes(n_q, ld_pools) + score_rows_bytes(n_q, ld_pools);
        rc = cuda_status(glm::launch_index_gemm(q_idx, w, static_cast<const float *>(keys), ld_pools, q_seq, q_pos, pad,
                                                len, batch, n_q, sbuf, scratch, status, sms, st));
        if (rc != GLM_OK) return rc;
        const glm::NvisSource src{nullptr, q_seq, q_pos, pad, len, batch, ld_pools};
        rc = cuda_status(glm::launch_topk_hist(sbuf, src, n_q, sw.hist, st));
        if (rc != GLM_OK) return rc;
        rc = cuda_status(glm::launch_topk_collect(sbuf, src, sw.hist, sw.hist2, sw.counters, sw.words, sw.alist,
                                                  sw.blist, n_q, select_k, topk, n_sel, st));
        if (rc != GLM_OK || (!tok && !rows)) return rc;
        return cuda_status(glm::launch_expand(topk, n_sel, q_seq, q_pos, pad, len, batch, n_q, select_k, slot_map,
                                              ld_slot, out_width, tok, rows, st));
    }
    if (zero && glm::index_select_ctas(n_q, ld_pools, sms) > 1) {
        const int rc = cuda_status(glm::launch_zero(sw.hist, align_up(sw.zero_bytes, 16), st));
        if (rc != GLM_OK) return rc;
    }
    glm::IxSelectArgs sel{};
    sel.select_k = select_k;
    sel.topk = topk;
    sel.n_sel = n_sel;
    sel.ghist = sw.hist;
    sel.ghist2 = sw.hist2;
    sel.counters = sw.counters;
    sel.words = sw.words;
    sel.alist = sw.alist;
    sel.blist = sw.blist;
    sel.list_cap = glm::sel_list_cap(ld_pools);
    sel.slot_map = slot_map;
    sel.ld_slot = ld_slot;
    sel.out_width = out_width;
    sel.tok = tok;
    sel.rows = rows;
    sel.gsamp = sw.fine;
    sel.early = new_pools >= 0 ? 1 : 0;   // new_pools < 0: wait for the preceding kernel at the start
    sel.new_pool_begin = new_pool_begin;
    sel.new_pools = new_pools >= 0 ? new_pools : 0;
    return cuda_status(glm::launch_index_select_tc(q_idx, w, keys, key_scales, ld_pools, q_seq, q_pos, pad, len, batch,
                                                   n_q, sbuf, scores != nullptr, sel, status, sms, st));
}

}  // namespace

int glm_index_scores_topk(const glm_dsa_dims *dims, const void *q_idx, const float *w,
                          const float *pooled, int64_t ld_pools, const int32_t *q_seq,
                          const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                          int32_t batch, int32_t n_q, int32_t select_k, float *scores,
                          int32_t *topk, int32_t *n_sel, void *workspace, size_t ws_bytes,
                          void *stream) {
    int rc = check_index_args(dims, q_idx, w, pooled, ld_pools, q_seq, q_pos, pad, len, batch, n_q, select_k,
                              scores, topk, n_sel);
    if (rc != GLM_OK || n_q == 0) return rc;
    return run_index_select(dims, q_idx, w, pooled, nullptr, ld_pools, q_seq, q_pos, pad, len, batch, n_q, select_k,
                            nullptr, 0, 0, scores, topk, n_sel, nullptr, nullptr, workspace, ws_bytes, stream);
}

int glm_index_topk_expand(const glm_dsa_dims *dims, const void *q_idx, const float *w,
                          const float *pooled, int64_t ld_pools, const int32_t *q_seq,
                          const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                          int32_t batch, int32_t n_q, int32_t select_k, const int64_t *slot_map,
                          int64_t ld_slot, int32_t out_width, float *scores, int32_t *topk,
                          int32_t *n_sel, int32_t *tok, int32_t *rows, void *workspace,
                          size_t ws_bytes, void *stream) {
    int rc = check_index_args(dims, q_idx, w, pooled, ld_pools, q_seq, q_pos, pad, len, batch, n_q, select_k,
                              scores, topk, n_sel);
    if (rc != GLM_OK) return rc;
    if (out_width < 1 || ld_slot < 0) return GLM_ERR_INVALID_ARG;
    if (static_cast<int64_t>(out_width) < static_cast<int64_t>(glm::kKpool) * select_k + glm::kKpool - 1)
        return GLM_ERR_INVALID_ARG;  // the largest selection plus a full tail must fit
    if (n_q == 0) return GLM_OK;
    if (!tok && !rows) return GLM_ERR_INVALID_ARG;
    if ((slot_map && !aligned(slot_map, 8)) || (tok && !aligned(tok, 4)) || (rows && !aligned(rows, 4)))
        return GLM_ERR_INVALID_ARG;
    return run_index_select(dims, q_idx, w, pooled, nullptr, ld_pools, q_seq, q_pos, pad, len, batch, n_q, select_k,
                            slot_map, ld_slot, out_width, scores, topk, n_sel, tok, rows, workspace, ws_bytes,
                            stream);
}

int glm_index_topk_expand_q8(const glm_dsa_dims *dims, const void *q_idx, const float *w,
                             const int8_t *pooled_codes, const float *pooled_scales, int64_t ld_pools,
                             const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                             int32_t batch, int32_t n_q, int32_t select_k, const int64_t *slot_map,
                             int64_t ld_slot, int32_t out_width, float *scores, int32_t *topk,
                             int32_t *n_sel, int32_t *tok, int32_t *rows, void *workspace,
                             size_t ws_bytes, void *stream) {
    int rc = check_index_args(dims, q_idx, w, pooled_codes, ld_pools, q_seq, q_pos, pad, len, batch, n_q, select_k,
                              scores, topk, n_sel);
    if (rc != GLM_OK) return rc;
    if (out_width < 1 || ld_slot < 0) return GLM_ERR_INVALID_ARG;
    if (static_cast<int64_t>(out_width) < static_cast<int64_t>(glm::kKpool) * select_k + glm::kKpool - 1)
        return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (!tok && !rows) return GLM_ERR_INVALID_ARG;
    if ((ld_pools > 0 && (!pooled_scales || !aligned(pooled_scales, 4))) || (slot_map && !aligned(slot_map, 8)) ||
        (tok && !aligned(tok, 4)) || (rows && !aligned(rows, 4)))
        return GLM_ERR_INVALID_ARG;
    return run_index_select(dims, q_idx, w, pooled_codes, pooled_scales ? pooled_scales : nullptr, ld_pools, q_seq,
                            q_pos, pad, len, batch, n_q, select_k, slot_map, ld_slot, out_width, scores, topk, n_sel,
                            tok, rows, workspace, ws_bytes, stream);
}

int glm_index_scores(const glm_dsa_dims *dims, const void *q_idx, const float *w,
                     const float *pooled, int64_t ld_pools, const int32_t *q_seq,
                     const int32_t *q_pos, const int32_t *pad, const int32_t *len, int32_t batch,
                     int32_t n_q, float *scores, void *stream) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_q < 0 || batch < 0 || ld_pools < 0 || n_q > 65535 || ld_pools > (int64_t(1) << 31) / 128)
        return GLM_ERR_INVALID_ARG;
    if (n_q == 0 || ld_pools == 0) return GLM_OK;
    if (batch == 0 || !q_idx || !w || !pooled || !q_seq || !q_pos || !pad || !len || !scores)
        return GLM_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(w, 4) || !aligned(pooled, 16) || !aligned(q_seq, 4) ||
        !aligned(q_pos, 4) || !aligned(pad, 4) || !aligned(len, 4) || !aligned(scores, 4))
        return GLM_ERR_INVALID_ARG;
    const glm::IxSelectArgs none{};   // topk == nullptr: scores only
    return cuda_status(glm::launch_index_select_tc(q_idx, w, pooled, nullptr, ld_pools, q_seq, q_pos, pad, len,
                                                   batch, n_q, scores, true, none, nullptr, num_sms(),
                                                   static_cast<cudaStream_t>(stream)));
}

int glm_topk_pools(const float *scores, int64_t ld_scores, const int32_t *n_visible, int32_t n_q,
                   int32_t select_k, int32_t *topk, int32_t *n_sel, void *workspace,
                   size_t ws_bytes, void *stream) {
    if (n_q < 0 || ld_scores < 0 || select_k < 1 || select_k > glm::kMaxSelect || n_q > 65535)
        return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (!n_visible || !topk || (ld_scores > 0 && !scores)) return GLM_ERR_INVALID_ARG;
    if ((scores && !aligned(scores, 4)) || !aligned(n_visible, 4) || !aligned(topk, 4) ||
        (n_sel && !aligned(n_sel, 4)))
        return GLM_ERR_INVALID_ARG;
    const size_t need = sel_bytes(n_q, ld_scores);
    if (workspace == nullptr || ws_bytes < need || !aligned(workspace, 256)) return GLM_ERR_WORKSPACE;
    const SelWs sw = sel_layout(workspace, n_q, ld_scores);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const glm::NvisSource src{n_visible, nullptr, nullptr, nullptr, nullptr, 0, ld_scores};
    int rc = cuda_status(glm::launch_zero(sw.hist, align_up(sw.zero_bytes, 16), st));
    if (rc != GLM_OK) return rc;
    rc = cuda_status(glm::launch_topk_hist(scores, src, n_q, sw.hist, st));
    if (rc != GLM_OK) return rc;
    return cuda_status(glm::launch_topk_collect(scores, src, sw.hist, sw.hist2, sw.counters, sw.words, sw.alist,
                                                sw.blist, n_q, select_k, topk, n_sel, st));
}

int glm_expand_selection(const glm_dsa_dims *dims, const int32_t *topk, const int32_t *n_sel,
                         const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad,
                         const int32_t *len, int32_t batch, int32_t n_q, int32_t select_k,
                         const int64_t *slot_map, int64_t ld_slot, int32_t out_width,
                         int32_t *tok, int32_t *rows, void *stream) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_q < 0 || batch < 0 || select_k < 1 || select_k > (1 << 24) || out_width < 1 || ld_slot < 0 ||
        n_q > 65535)
        return GLM_ERR_INVALID_ARG;
    if (static_cast<int64_t>(out_width) < static_cast<int64_t>(glm::kKpool) * select_k + glm::kKpool - 1)
        return GLM_ERR_INVALID_ARG;  // the largest selection plus a full tail must fit
    if (n_q == 0) return GLM_OK;
    if (batch == 0 || !topk || !q_seq || !q_pos || !pad || !len || (!tok && !rows)) return GLM_ERR_INVALID_ARG;
    if (!aligned(topk, 4) || (n_sel && !aligned(n_sel, 4)) || !aligned(q_seq, 4) ||
        !aligned(q_pos, 4) || !aligned(pad, 4) || !aligned(len, 4) ||
        (slot_map && !aligned(slot_map, 8)) || (tok && !aligned(tok, 4)) || (rows && !aligned(rows, 4)))
        return GLM_ERR_INVALID_ARG;
    return cuda_status(glm::launch_expand(topk, n_sel, q_seq, q_pos, pad, len, batch, n_q, select_k,
                                          slot_map, ld_slot, out_width, tok, rows,
                                          static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {
// The split + combine of one sparse MLA call over rows of the given format.
int sparse_mla_entry(const glm_dsa_dims *dims, const void *q, const int8_t *cache, int64_t n_rows,
                     const int32_t *rows, int32_t n_q, int32_t width, float sm_scale, void *out, float *lse,
                     float *out_f32, void *workspace, size_t ws_bytes, void *stream, int format) {
    int rc = check_mla(dims, q, cache, n_rows, rows, n_q, width, sm_scale, out, lse, out_f32);
    if (rc != GLM_OK || n_q == 0) return rc;
    const int H = dims->n_heads;
    const size_t need = glm_dsa_workspace_size(dims, GLM_OP_SPARSE_MLA, n_q, 0, 0, width);
    if (workspace == nullptr || ws_bytes < need || !aligned(workspace, 256)) return GLM_ERR_WORKSPACE;
    const glm::MlaPlan plan = glm::mla_plan(n_q, H, width, num_sms());
    const size_t parts = mla_parts(n_q, H, width);
    char *ws = static_cast<char *>(workspace);
    float *part_acc = reinterpret_cast<float *>(ws);
    float *part_ml = reinterpret_cast<float *>(ws + mla_acc_bytes(parts));
    int *status = reinterpret_cast<int *>(ws + mla_acc_bytes(parts) + mla_ml_bytes(parts));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = cuda_status(glm::launch_mla_split_tc(plan, q, H, cache, n_rows, rows, n_q, width, sm_scale, part_acc, part_ml,
                                              status, st, false, format, out, out_f32, lse));
    if (rc != GLM_OK || !plan.combine) return rc;
    return cuda_status(glm::launch_mla_combine(part_acc, part_ml, n_q, H, plan.n_parts, out, out_f32, lse, st));
}
}  // namespace

extern "C" {

int glm_sparse_mla_decode(const glm_dsa_dims *dims, const void *q, const int8_t *cache,
                          int64_t n_rows, const int32_t *rows, int32_t n_q, int32_t width,
                          float sm_scale, void *out, float *lse, float *out_f32, void *workspace,
                          size_t ws_bytes, void *stream) {
    return sparse_mla_entry(dims, q, cache, n_rows, rows, n_q, width, sm_scale, out, lse, out_f32, workspace,
                            ws_bytes, stream, glm::kFmtInt8);
}

int glm_sparse_mla_decode_fp8(const glm_dsa_dims *dims, const void *q, const uint8_t *cache,
                              int64_t n_rows, const int32_t *rows, int32_t n_q, int32_t width,
                              float sm_scale, void *out, float *lse, float *out_f32, void *workspace,
                              size_t ws_bytes, void *stream) {
    return sparse_mla_entry(dims, q, reinterpret_cast<const int8_t *>(cache), n_rows, rows, n_q, width, sm_scale,
                            out, lse, out_f32, workspace, ws_bytes, stream, glm::kFmtFp8);
}

int glm_sparse_mla_decode_fp4(const glm_dsa_dims *dims, const void *q, const uint8_t *cache,
                              int64_t n_rows, const int32_t *rows, int32_t n_q, int32_t width,
                              float sm_scale, void *out, float *lse, float *out_f32, void *workspace,
                              size_t ws_bytes, void *stream) {
    return sparse_mla_entry(dims, q, reinterpret_cast<const int8_t *>(cache), n_rows, rows, n_q, width, sm_scale,
                            out, lse, out_f32, workspace, ws_bytes, stream, glm::kFmtFp4);
}

int glm_cp_candidates(const float *scores, int64_t ld_scores, const int32_t *topk, int32_t n_q, int32_t select_k,
                      int32_t rank, int32_t world, float *cand_scores, int32_t *cand_ids, void *stream) {
    if (n_q < 0 || n_q > 65535 || ld_scores < 0 || select_k < 1 || select_k > glm::kMaxSelect || world < 1 ||
        rank < 0 || rank >= world || ld_scores > (int64_t(1) << 31) / world)
        return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if ((ld_scores > 0 && !scores) || !topk || !cand_scores || !cand_ids) return GLM_ERR_INVALID_ARG;
    if ((scores && !aligned(scores, 4)) || !aligned(topk, 4) || !aligned(cand_scores, 4) || !aligned(cand_ids, 4))
        return GLM_ERR_INVALID_ARG;
    return cuda_status(glm::launch_cp_candidates(scores, ld_scores, topk, n_q, select_k, rank, world, cand_scores,
                                                 cand_ids, static_cast<cudaStream_t>(stream)));
}

int glm_merge_topk(const float *cand_scores, const int32_t *cand_ids, int32_t n_parts, int32_t n_q, int32_t per_part,
                   int32_t select_k, int32_t *topk, int32_t *n_sel, void *stream) {
    if (n_parts < 1 || n_q < 0 || n_q > 65535 || per_part < 0 || select_k < 1 || select_k > glm::kMaxSelect ||
        static_cast<int64_t>(n_parts) * per_part > (int64_t(1) << 24))
        return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (!topk || (per_part > 0 && (!cand_scores || !cand_ids))) return GLM_ERR_INVALID_ARG;
    if ((cand_scores && !aligned(cand_scores, 4)) || (cand_ids && !aligned(cand_ids, 4)) || !aligned(topk, 4) ||
        (n_sel && !aligned(n_sel, 4)))
        return GLM_ERR_INVALID_ARG;
    return cuda_status(glm::launch_merge_topk(cand_scores, cand_ids, n_parts, n_q, per_part, select_k, topk, n_sel,
                                              static_cast<cudaStream_t>(stream)));
}

int glm_lse_merge(const glm_dsa_dims *dims, const float *out_parts, const float *lse_parts, int32_t n_parts,
                  int32_t n_q, void *out, float *out_f32, float *lse, void *stream) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_parts < 1 || n_q < 0 || n_q > 65535) return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (!out_parts || !lse_parts || !out) return GLM_ERR_INVALID_ARG;
    if (!aligned(out_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16) || (out_f32 && !aligned(out_f32, 16)) ||
        (lse && !aligned(lse, 4)))
        return GLM_ERR_INVALID_ARG;
    return cuda_status(glm::launch_lse_merge(out_parts, lse_parts, n_parts, n_q, dims->n_heads, out, out_f32, lse,
                                             static_cast<cudaStream_t>(stream)));
}

int glm_mla_v_up(const glm_dsa_dims *dims, const void *o_lat, const void *w_kv_b, int32_t qk_nope_head_dim,
                 int32_t v_head_dim, int32_t n_q, void *out_v, float *out_v_f32, void *stream) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_q < 0 || n_q > 65535 * 128 || qk_nope_head_dim < 0 || v_head_dim < 128 || v_head_dim % 128 != 0 ||
        v_head_dim > 4096 || qk_nope_head_dim > 4096)
        return GLM_ERR_INVALID_ARG;
    if (static_cast<int64_t>(dims->n_heads) * (qk_nope_head_dim + v_head_dim) > (int64_t(1) << 31))
        return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (!o_lat || !w_kv_b || !out_v) return GLM_ERR_INVALID_ARG;
    if (!aligned(o_lat, 16) || !aligned(w_kv_b, 16) || !aligned(out_v, 16) || (out_v_f32 && !aligned(out_v_f32, 16)))
        return GLM_ERR_INVALID_ARG;
    return cuda_status(glm::launch_mla_vup(o_lat, w_kv_b, dims->n_heads, qk_nope_head_dim, v_head_dim, n_q, out_v,
                                           out_v_f32, static_cast<cudaStream_t>(stream)));
}

int glm_dsa_decode_step(const glm_dsa_dims *dims, const glm_dsa_step *a, void *workspace, size_t ws_bytes,
                        void *stream) {
    if (a == nullptr) return GLM_ERR_INVALID_ARG;
    if (a->cache_format < GLM_CACHE_INT8 || a->cache_format > GLM_CACHE_FP4) return GLM_ERR_INVALID_ARG;
    const bool q8 = a->pooled_codes_dev != nullptr;   // the INT8 indexer state replaces pooled_dev
    const void *keys = q8 ? static_cast<const void *>(a->pooled_codes_dev) : static_cast<const void *>(a->pooled_dev);
    if (q8 && (!a->pooled_scales_dev || !aligned(a->pooled_scales_dev, 4))) return GLM_ERR_INVALID_ARG;
    int rc = check_store(dims, a->latent_dev, a->slots_dev, a->n_new, a->cache_dev, a->n_rows);
    if (rc != GLM_OK) return rc;
    rc = check_kpool(dims, a->k_dev, a->gate_dev, a->ld_tokens, a->ln_w_dev, a->ln_b_dev, a->ln_eps, a->pad_dev,
                     a->len_dev, a->pool_begin_dev, a->batch, a->max_new_pools, keys, a->ld_pools, nullptr);
    if (rc != GLM_OK) return rc;
    rc = check_index_args(dims, a->q_idx_dev, a->w_dev, keys, a->ld_pools, a->q_seq_dev, a->q_pos_dev,
                          a->pad_dev, a->len_dev, a->batch, a->n_q, a->select_k, a->scores_dev, a->topk_dev,
                          a->n_sel_dev);
    if (rc != GLM_OK) return rc;
    if (a->out_width < 1 || a->ld_slot < 0 ||
        static_cast<int64_t>(a->out_width) < static_cast<int64_t>(glm::kKpool) * a->select_k + glm::kKpool - 1)
        return GLM_ERR_INVALID_ARG;
    if (a->n_q > 0 && !a->rows_dev) return GLM_ERR_INVALID_ARG;   // the attention reads them
    if ((a->slot_map_dev && !aligned(a->slot_map_dev, 8)) || (a->tok_dev && !aligned(a->tok_dev, 4)) ||
        (a->rows_dev && !aligned(a->rows_dev, 4)))
        return GLM_ERR_INVALID_ARG;
    rc = check_mla(dims, a->q_dev, a->cache_dev, a->n_rows, a->rows_dev, a->n_q, a->out_width, a->sm_scale,
                   a->out_dev, a->lse_dev, a->out_f32_dev);
    if (rc != GLM_OK) return rc;
    const StepLayout L = step_layout(dims, a->n_q, a->ld_pools, a->out_width);
    if (workspace == nullptr || ws_bytes < L.total || !aligned(workspace, 256)) return GLM_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    int *status = reinterpret_cast<int *>(ws + L.total - 256);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int sms = num_sms();
    const bool idx_multi = a->n_q > 0 && (index_by_gemm(a->n_q, a->ld_pools, a->batch, q8) ||
                                          glm::index_select_ctas(a->n_q, a->ld_pools, sms) > 1);
    const SelWs sw = sel_layout(ws + L.idx, a->n_q, a->ld_pools);
    glm::StepPrepArgs p{};
    p.latent = static_cast<const uint16_t *>(a->latent_dev);
    p.slots = a->slots_dev;
    p.n_new = a->n_new;
    p.cache = a->cache_dev;
    p.n_rows = a->n_rows;
    p.k = static_cast<const uint16_t *>(a->k_dev);
    p.gate = static_cast<const uint16_t *>(a->gate_dev);
    p.ld_tokens = a->ld_tokens;
    p.ln_w = a->ln_w_dev;
    p.ln_b = a->ln_b_dev;
    p.ln_eps = a->ln_eps;
    p.pad = a->pad_dev;
    p.len = a->len_dev;
    p.pool_begin = a->pool_begin_dev;
    p.batch = a->batch;
    p.max_new_pools = a->max_new_pools;
    p.pooled = q8 ? nullptr : a->pooled_dev;
    p.codes = q8 ? a->pooled_codes_dev : nullptr;
    p.scales = q8 ? a->pooled_scales_dev : nullptr;
    p.ld_pools = a->ld_pools;
    p.format = a->cache_format;
    p.zero = reinterpret_cast<uint4 *>(sw.hist);
    p.zero_n16 = idx_multi ? static_cast<int64_t>(align_up(sw.zero_bytes, 16) / 16) : 0;
    if (a->stop_after < 0 || a->stop_after > 3) return GLM_ERR_INVALID_ARG;
    rc = cuda_status(glm::launch_step_prep(p, st));
    if (rc != GLM_OK || a->n_q == 0 || a->stop_after == 1) return rc;
    rc = enqueue_index_select(a->q_idx_dev, a->w_dev, keys, q8 ? a->pooled_scales_dev : nullptr, a->ld_pools,
                              a->q_seq_dev, a->q_pos_dev,
                              a->pad_dev, a->len_dev, a->batch, a->n_q, a->select_k, a->slot_map_dev, a->ld_slot,
                              a->out_width, a->scores_dev, a->topk_dev, a->n_sel_dev, a->tok_dev, a->rows_dev,
                              ws + L.idx, status, false, sms, st, a->pool_begin_dev,
                              a->batch > 0 ? a->max_new_pools : 0);
    if (rc != GLM_OK || a->stop_after == 2) return rc;
    const int H = dims->n_heads;
    const glm::MlaPlan plan = glm::mla_plan(a->n_q, H, a->out_width, sms);
    const size_t parts = mla_parts(a->n_q, H, a->out_width);
    float *part_acc = reinterpret_cast<float *>(ws + L.mla);
    float *part_ml = reinterpret_cast<float *>(ws + L.mla + mla_acc_bytes(parts));
    rc = cuda_status(glm::launch_mla_split_tc(plan, a->q_dev, H, a->cache_dev, a->n_rows, a->rows_dev, a->n_q, a->out_width,
                                              a->sm_scale, part_acc, part_ml, status, st, true, a->cache_format,
                                              a->out_dev, a->out_f32_dev, a->lse_dev));
    if (rc != GLM_OK || a->stop_after == 3 || !plan.combine) return rc;
    return cuda_status(glm::launch_mla_combine(part_acc, part_ml, a->n_q, H, plan.n_parts, a->out_dev, a->out_f32_dev,
                                               a->lse_dev, st));
}

}  // extern "C"
