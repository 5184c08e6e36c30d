// sparse_mla.cuh -- launchers of the sparse NoPE MLA split and combine kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace glm {

// Partial softmax state of one (query, part, head): m (max of the part's scores), l (sum of
// exp(s - m)), acc[512] (sum of exp(s - m) * c). Layout in the workspace:
//   part_acc fp32 [n_q][n_parts][n_heads][512], part_ml fp32 [n_q][n_parts][n_heads][2].
// mla_tc_chunk(): the entries of one chunk in every plan.
int mla_tc_chunk();

// How the attention cuts the work: chunks of `rows` index entries, groups of `heads` heads.
// Few queries (multi false): one CTA per (query, chunk, head group), one partial per chunk
// (n_parts = n_chunks). Many queries (multi true): one CTA per (query, run of cpc chunks, head
// group) walking its chunks, one partial per run (n_parts runs); with one run (combine false)
// that CTA writes the final output itself and no combine follows.
struct MlaPlan {
    int rows, heads, n_chunks, n_hg;
    int cpc, n_parts;
    bool multi, combine;
};
MlaPlan mla_plan(int n_q, int n_heads, int width, int num_sms);
// The largest query count that takes the few-query plan (at least two CTAs per SM above it).
long long mla_few_query_max(int n_heads, int num_sms);

// The split kernel of the plan: partials [n_q][plan.n_parts][n_heads] (then launch_mla_combine
// with n_chunks = plan.n_parts), or, when plan.combine is false, out / out_f32 / lse directly.
cudaError_t launch_mla_split_tc(const MlaPlan &plan, const void *q, int n_heads, const int8_t *cache, int64_t n_rows,
                                const int32_t *rows, int n_q, int width, float sm_scale,
                                float *part_acc, float *part_ml, int *status, cudaStream_t stream,
                                bool early_q = false,    // early_q: stage q before waiting on the previous kernel
                                int format = 0,          // CacheFormat of the rows (int8, fp8 or 4-bit)
                                void *out = nullptr, float *out_f32 = nullptr, float *lse = nullptr);
// poison (or null): a status word the split kernel sets on a timed-out wait; when it is nonzero
// the combine writes NaN to every output instead of merging (used where the caller cannot read it).
cudaError_t launch_mla_combine(const float *part_acc, const float *part_ml, int n_q, int n_heads,
                               int n_chunks, void *out, float *out_f32, float *lse,
                               cudaStream_t stream, const int *poison = nullptr);

}  // namespace glm
