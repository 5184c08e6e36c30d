// sparse_mla.cuh -- launchers of the sparse NoPE MLA split and combine kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace glm {

// Partial softmax state of one (query, chunk, head): m (max of the chunk's scores), l (sum of
// exp(s - m)), acc[512] (sum of exp(s - m) * c). Layout in the workspace:
//   part_acc fp32 [n_q][n_chunks][n_heads][512], part_ml fp32 [n_q][n_chunks][n_heads][2].
// mla_tc_chunk(): the smallest chunk of any plan (workspaces are sized for it).
int mla_tc_chunk();

// How the split kernel cuts the work: chunks of `rows` index entries, groups of `heads` heads.
struct MlaPlan {
    int rows, heads, n_chunks, n_hg;
};
MlaPlan mla_plan(int n_q, int n_heads, int width, int num_sms);

cudaError_t launch_mla_split_tc(const MlaPlan &plan, const void *q, int n_heads, const int8_t *cache, int64_t n_rows,
                                const int32_t *rows, int n_q, int width, float sm_scale,
                                float *part_acc, float *part_ml, int *status, cudaStream_t stream,
                                bool early_q = false,    // early_q: stage q before waiting on the previous kernel
                                int format = 0);         // CacheFormat of the rows (int8, fp8 or 4-bit)
// poison (or null): a status word the split kernel sets on a timed-out wait; when it is nonzero
// the combine writes NaN to every output instead of merging (used where the caller cannot read it).
cudaError_t launch_mla_combine(const float *part_acc, const float *part_ml, int n_q, int n_heads,
                               int n_chunks, void *out, float *out_f32, float *lse,
                               cudaStream_t stream, const int *poison = nullptr);

}  // namespace glm
