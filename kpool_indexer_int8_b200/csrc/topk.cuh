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

// Warp-aggregated add of one digit per lane into a shared histogram (0xffffffff = no digit).
// Every lane of the warp must call it.
__device__ __forceinline__ void hist_add(unsigned *hist, uint32_t digit) {
    const unsigned peers = __match_any_sync(0xffffffffu, digit);
    if (digit != 0xffffffffu && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
}

// Workspace of a selection, per query: the histogram (kHistBins uint32) and four uint32
// counters (list A size, list B size, finished CTAs) -- both zeroed before each selection --,
// list A (kMaxSelect uint64 composites) and list B (ld uint64 composites).
size_t topk_select_smem();
cudaError_t launch_zero(void *p, size_t bytes, cudaStream_t stream);   // p 16-byte aligned
int topk_collect_ctas(int64_t ld);
cudaError_t launch_topk_hist(const float *scores, const NvisSource &src, int n_q, unsigned *ghist,
                             cudaStream_t stream);
cudaError_t launch_topk_collect(const float *scores, const NvisSource &src, const unsigned *ghist,
                                unsigned *counters, unsigned long long *alist,
                                unsigned long long *blist, int n_q, int select_k, int32_t *topk,
                                int32_t *n_sel, cudaStream_t stream);

}  // namespace glm
