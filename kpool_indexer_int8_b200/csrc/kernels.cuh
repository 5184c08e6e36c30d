// kernels.cuh -- launchers behind the C ABI (one per kernel family).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "glm_dsa.h"
#include "sparse_mla.cuh"
#include "topk.cuh"

namespace glm {

// Host helpers of the C ABI shared by its source files.
namespace abi {
int cuda_status(cudaError_t e);   // GLM_OK, or GLM_ERR_CUDA with e kept for glm_last_cuda_error()
int num_sms();                    // SMs of the current device
int check_mla(const glm_dsa_dims *dims, const void *q, const int8_t *cache, int64_t n_rows, const int32_t *rows,
              int32_t n_q, int32_t width, float sm_scale, const void *out, const float *lse, const float *out_f32);
}  // namespace abi

cudaError_t launch_store_int8(const void *latent, const int64_t *slots, int64_t n, int8_t *cache,
                              int64_t n_rows, cudaStream_t stream, int num_sms);
cudaError_t launch_store_fp8(const void *latent, const int64_t *slots, int64_t n, uint8_t *cache,
                             int64_t n_rows, cudaStream_t stream, int num_sms);
cudaError_t launch_store_fp4(const void *latent, const int64_t *slots, int64_t n, uint8_t *cache,
                             int64_t n_rows, cudaStream_t stream, int num_sms);
cudaError_t launch_kpool_build(const void *k, const void *gate, int64_t ld_tokens,
                               const float *ln_w, const float *ln_b, float eps,
                               const int32_t *pad, const int32_t *len, const int32_t *pool_begin,
                               int batch, int max_new_pools, float *pooled, int64_t ld_pools,
                               int32_t *n_pools, cudaStream_t stream, int num_sms,
                               int8_t *codes = nullptr, float *scales = nullptr);   // codes: INT8 state
// Selection and expansion arguments of the fused index kernel; topk == nullptr: scores only.
// The multi-CTA counters (kCntWords uint32 per query) must be zero at launch when
// index_select_ctas() > 1 (or be zeroed by the kernel launched just before it, which the kernel
// waits for before it touches them); gsamp (kSampleUnion uint32 per query, 16-byte aligned) needs
// no zeroing. ghist and ghist2 are not used by this kernel.
struct IxSelectArgs {
    int select_k;
    int32_t *topk;                 // [n_q][select_k]
    int32_t *n_sel;                // [n_q] or null
    unsigned *ghist;               // [n_q][kHistBins] level-1 histograms
    unsigned *ghist2;              // [n_q][kHistBins] level-2 histograms
    unsigned *gsamp;               // [n_q][kSampleUnion] sample keys published by the CTAs
    unsigned *counters;            // [n_q][kCntWords]
    unsigned *words;               // [n_q][kMaxSelCtas] list sizes of each CTA
    unsigned long long *alist;     // [n_q][list_cap] per-CTA regions of list A
    unsigned long long *blist;     // [n_q][list_cap] per-CTA regions of list B
    long long list_cap;            // sel_list_cap(ld_pools)
    const int64_t *slot_map;       // expansion: [batch][ld_slot] or null
    long long ld_slot;
    int out_width;
    int32_t *tok;                  // [n_q][out_width] or null
    int32_t *rows;                 // [n_q][out_width] or null
    // early != 0 (one-call step): the preceding kernel writes only pooled rows [new_pool_begin[b],
    // + new_pools) of each sequence b (plus buffers this kernel does not read before it waits), so
    // the kernel streams every other pooled key before waiting for it
    int early;
    const int32_t *new_pool_begin; // [batch] or null (= 0)
    int new_pools;
};
int index_select_ctas(int n_q, int64_t ld_pools, int num_sms);

// Scores of many queries at once (index_gemm.cu): queries of one sequence share the converted
// pooled keys; scratch of index_gemm_scratch_bytes(n_q) bytes, 256-byte aligned. Every score of
// rows [0, n_q) x [0, ld_pools) is written (-inf past the query's visible pools).
constexpr int kIndexGemmMinQueries = 128;   // fp32 keys and at least this many queries: the GEMM path
size_t index_gemm_scratch_bytes(int n_q);
cudaError_t launch_index_gemm(const void *q_idx, const float *w, const float *pooled, int64_t ld_pools,
                              const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                              int batch, int n_q, float *scores, void *scratch, int *status, int num_sms,
                              cudaStream_t stream);
cudaError_t set_cross_cta_wait_limit(uint32_t polls);   // the index kernel's meetings (current device)
cudaError_t launch_index_select_tc(const void *q_idx, const float *w, const void *keys,
                                   const float *key_scales, int64_t ld_pools, const int32_t *q_seq,
                                   const int32_t *q_pos, const int32_t *pad, const int32_t *len, int batch,
                                   int n_q, float *scores, bool fill_invisible, const IxSelectArgs &sel,
                                   int *status, int num_sms, cudaStream_t stream);   // key_scales: INT8 keys
// The fused step's first kernel: store rows, build pools, zero a word range (16-byte units).
struct StepPrepArgs {
    const uint16_t *latent;
    const int64_t *slots;
    int64_t n_new;
    int8_t *cache;
    int64_t n_rows;
    const uint16_t *k;
    const uint16_t *gate;
    int64_t ld_tokens;
    const float *ln_w;
    const float *ln_b;
    float ln_eps;
    const int32_t *pad;
    const int32_t *len;
    const int32_t *pool_begin;
    int batch;
    int max_new_pools;
    float *pooled;
    int8_t *codes;                 // INT8 indexer state (pooled unused) or null
    float *scales;
    int64_t ld_pools;
    uint4 *zero;
    int64_t zero_n16;
    int format;                    // CacheFormat of the cache rows
};
cudaError_t launch_step_prep(const StepPrepArgs &a, cudaStream_t stream);

// The up-projection after the absorbed MLA (mla_vup.cu): out_v = o_lat . W_v,h^T per head.
cudaError_t launch_mla_vup(const void *o_lat, const void *w_kv_b, int n_heads, int dk, int dv, int n_q, void *out_v,
                           float *out_f32, cudaStream_t stream);

// Context parallelism: a rank's selection as (score, global pool id) candidates; the global top-k
// of every rank's candidates ([n_parts][n_q][per_part]); the log-sum-exp merge of attention parts.
cudaError_t launch_cp_candidates(const float *scores, int64_t ld, const int32_t *topk, int n_q, int select_k,
                                 int rank, int world, float *cand_scores, int32_t *cand_ids, cudaStream_t stream);
cudaError_t launch_merge_topk(const float *cand_scores, const int32_t *cand_ids, int n_parts, int n_q, int per_part,
                              int select_k, int32_t *topk, int32_t *n_sel, cudaStream_t stream);
cudaError_t launch_lse_merge(const float *out_parts, const float *lse_parts, int n_parts, int n_q, int n_heads,
                             void *out, float *out_f32, float *lse, cudaStream_t stream);

cudaError_t launch_expand(const int32_t *topk, const int32_t *n_sel, const int32_t *q_seq,
                          const int32_t *q_pos, const int32_t *pad, const int32_t *len, int batch,
                          int n_q, int select_k, const int64_t *slot_map, int64_t ld_slot, int out_width,
                          int32_t *tok, int32_t *rows, cudaStream_t stream);

}  // namespace glm
