// topk.cuh -- launchers of the top-k selection kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace glm {

constexpr int kHistBitsTop = 11;                 // histogram over the top 11 bits of a score key
constexpr int kHistBins = 1 << kHistBitsTop;

// Where a query's visible-pool count comes from: an explicit array (scores-in entry) or the
// sequence geometry (fused entry); ld = leading dimension of the score rows (and the cap).
struct NvisSource {
    const int32_t *n_visible;
    const int32_t *q_seq;
    const int32_t *q_pos;
    const int32_t *pad;
    const int32_t *len;
    int batch;
    long long ld;
};

// Workspace of a selection, per query: two histograms (kHistBins uint32 each) and kCntWords
// uint32 counters -- all zeroed before each selection --, kMaxSelCtas uint32 list sizes, and the
// per-CTA regions of list A and list B (sel_list_cap(ld) uint64 composites each).
size_t topk_select_smem();
cudaError_t launch_zero(void *p, size_t bytes, cudaStream_t stream);   // p 16-byte aligned
int topk_collect_ctas(int64_t ld);
cudaError_t launch_topk_hist(const float *scores, const NvisSource &src, int n_q, unsigned *ghist,
                             cudaStream_t stream);
cudaError_t launch_topk_collect(const float *scores, const NvisSource &src, const unsigned *ghist,
                                unsigned *ghist2, unsigned *counters, unsigned *words, unsigned long long *alist,
                                unsigned long long *blist, int n_q, int select_k, int32_t *topk,
                                int32_t *n_sel, cudaStream_t stream);

}  // namespace glm
