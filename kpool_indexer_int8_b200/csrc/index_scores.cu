// index_scores.cu -- relu head-weighted index scores ("Module glm5next_dsa_ref", index_scores:
// the matmul -> relu -> head-weighted sum chain; "GLM-5.3-Flash" pypto-lib page: indexer
// 32 heads x 128):
//     score[n][p] = sum_h w[n][h] * max(0, sum_d q_idx[n][h][d] * pooled[b][p][d])
//
// SIMT form: one thread per pool, 32 fp32 accumulators per thread, the query's 32 x 128 indexer
// query widened to fp32 in shared memory and read as broadcast float4. Entries p >= n_vis of the
// score row are written as -inf. HBM-bound on the pooled keys (512 bytes per pool) but limited
// by FFMA issue (4096 FMAs per pool); the tensor-core kernel replaces it on the hot path.
#include "common.cuh"
#include "topk.cuh"

namespace glm {

constexpr int kScoreThreads = 128;

__global__ void __launch_bounds__(kScoreThreads) index_scores_simt_kernel(
    const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
    const float *__restrict__ pooled, int64_t ld_pools, const int32_t *__restrict__ q_seq,
    const int32_t *__restrict__ q_pos, const int32_t *__restrict__ pad,
    const int32_t *__restrict__ len, int batch, float *__restrict__ scores,
    unsigned *__restrict__ ghist) {
    __shared__ __align__(16) float qs[kIdxHeads][kIdxDim];
    __shared__ float ws[kIdxHeads];
    __shared__ unsigned hist[kHistBins];
    const int n = blockIdx.y;
    const int b = q_seq[n];
    const int n_vis = (b >= 0 && b < batch) ? visible_pools(pad[b], len[b], q_pos[n], ld_pools) : 0;
    const int64_t p = static_cast<int64_t>(blockIdx.x) * kScoreThreads + threadIdx.x;
    float *srow = scores + static_cast<int64_t>(n) * ld_pools;
    if (static_cast<int64_t>(blockIdx.x) * kScoreThreads >= n_vis) {  // whole block invisible
        if (p < ld_pools) srow[p] = -INFINITY;
        return;
    }
    const uint16_t *qn = q_idx + static_cast<int64_t>(n) * kIdxHeads * kIdxDim;
    for (int i = threadIdx.x; i < kIdxHeads * kIdxDim; i += kScoreThreads)
        (&qs[0][0])[i] = bf16_bits_to_float(qn[i]);
    if (threadIdx.x < kIdxHeads) ws[threadIdx.x] = w[static_cast<int64_t>(n) * kIdxHeads + threadIdx.x];
    if (ghist)
        for (int i = threadIdx.x; i < kHistBins; i += kScoreThreads) hist[i] = 0;
    __syncthreads();
    uint32_t digit = 0xffffffffu;
    if (p < n_vis) {
        const float4 *kp = reinterpret_cast<const float4 *>(pooled + (static_cast<int64_t>(b) * ld_pools + p) * kIdxDim);
        float acc[kIdxHeads];
#pragma unroll
        for (int h = 0; h < kIdxHeads; h++) acc[h] = 0.0f;
#pragma unroll 2
        for (int d4 = 0; d4 < kIdxDim / 4; d4++) {
            const float4 kv = __ldg(kp + d4);
#pragma unroll
            for (int h = 0; h < kIdxHeads; h++) {
                const float4 qv = reinterpret_cast<const float4 *>(qs[h])[d4];
                acc[h] = fmaf(qv.x, kv.x, acc[h]);
                acc[h] = fmaf(qv.y, kv.y, acc[h]);
                acc[h] = fmaf(qv.z, kv.z, acc[h]);
                acc[h] = fmaf(qv.w, kv.w, acc[h]);
            }
        }
        float sc = 0.0f;
#pragma unroll
        for (int h = 0; h < kIdxHeads; h++) sc = fmaf(ws[h], fmaxf(acc[h], 0.0f), sc);
        srow[p] = sc;
        digit = score_key(sc) >> (32 - kHistBitsTop);
    } else if (p < ld_pools) {
        srow[p] = -INFINITY;
    }
    if (ghist) {
        hist_add(hist, digit);
        __syncthreads();
        unsigned *g = ghist + static_cast<int64_t>(n) * kHistBins;
        for (int i = threadIdx.x; i < kHistBins; i += kScoreThreads)
            if (hist[i]) atomicAdd(&g[i], hist[i]);
    }
}

cudaError_t launch_index_scores_simt(const void *q_idx, const float *w, const float *pooled,
                                     int64_t ld_pools, const int32_t *q_seq, const int32_t *q_pos,
                                     const int32_t *pad, const int32_t *len, int batch, int n_q,
                                     float *scores, unsigned *ghist, cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>((ld_pools + kScoreThreads - 1) / kScoreThreads), n_q);
    index_scores_simt_kernel<<<grid, kScoreThreads, 0, stream>>>(
        static_cast<const uint16_t *>(q_idx), w, pooled, ld_pools, q_seq, q_pos, pad, len, batch,
        scores, ghist);
    return cudaGetLastError();
}

}  // namespace glm
