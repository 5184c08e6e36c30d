// topk.cu -- selection of the select_k highest-scoring visible pools on given scores ("Module
// glm5next_dsa_ref", topk_pools), ordered by score descending with ties to the lower pool id.
//
//   1. topk_hist_kernel: the level-1 histogram (top 11 key bits) of every query's scores;
//   2. topk_collect_kernel, grid (C, n_q): each CTA classifies a slice of the scores against the
//      boundary bin into list A / list B (level-2 digits counted in global memory); with C > 1 the
//      lists are appended to the query's global lists and the last CTA to finish (ticket)
//      completes the selection (select.cuh), sorts it and writes the row.
// The fused score kernel (index_select_tc.cu) runs the same selection without the score round trip.
#include "common.cuh"
#include "select.cuh"
#include "topk.cuh"

namespace glm {

constexpr int kCollectThreads = 512;

__device__ __forceinline__ int nvis_of(const NvisSource &s, int n) {
    if (s.n_visible) {
        long long v = s.n_visible[n];
        if (v < 0) v = 0;
        if (v > s.ld) v = s.ld;
        return static_cast<int>(v);
    }
    const int b = s.q_seq[n];
    if (b < 0 || b >= s.batch) return 0;
    return visible_pools(s.pad[b], s.len[b], s.q_pos[n], s.ld);
}

// ------------------------------------------------------------------------------------------------
// level-1 histogram of caller-supplied scores: grid (chunks of 8192 scores, n_q), 256 threads
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_hist_kernel(const float *__restrict__ scores, NvisSource src,
                                                        unsigned *__restrict__ ghist) {
    pdl_begin();
    __shared__ unsigned hist[kHistBins];
    const int n = blockIdx.y;
    const int n_vis = nvis_of(src, n);
    const int64_t lo = static_cast<int64_t>(blockIdx.x) * 8192;
    if (lo >= n_vis) return;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const float *row = scores + static_cast<int64_t>(n) * src.ld;
#pragma unroll 4
    for (int u = 0; u < 32; u++) {
        const int64_t i = lo + u * 256 + threadIdx.x;
        if (i < n_vis) atomicAdd(&hist[score_key(__ldg(row + i)) >> (32 - kHistBitsTop)], 1u);
    }
    __syncthreads();
    unsigned *g = ghist + static_cast<int64_t>(n) * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
        if (hist[i]) atomicAdd(&g[i], hist[i]);
}

// ------------------------------------------------------------------------------------------------
// selection kernel
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kCollectThreads) topk_collect_kernel(
    const float *__restrict__ scores, NvisSource src, const unsigned *__restrict__ ghist,
    unsigned *__restrict__ ghist2, unsigned *__restrict__ counters, unsigned *__restrict__ words,
    unsigned long long *__restrict__ alist, unsigned long long *__restrict__ blist, int64_t list_cap, int select_k,
    int32_t *__restrict__ topk, int32_t *__restrict__ n_sel_out) {
    pdl_begin();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SelShared &s = *reinterpret_cast<SelShared *>(smem_raw);
    __shared__ __align__(16) unsigned hist[kHistBins];
    const int n = blockIdx.y, c = blockIdx.x, C = gridDim.x;
    const int tid = threadIdx.x;
    const int n_vis = nvis_of(src, n);
    const float *row = scores + static_cast<int64_t>(n) * src.ld;
    int32_t *out = topk + static_cast<int64_t>(n) * select_k;
    const unsigned count = static_cast<unsigned>(min(select_k, n_vis));
    if (n_vis == 0) {
        if (c == 0) {
            write_selection(out, select_k, 0u, s);
            if (tid == 0 && n_sel_out) n_sel_out[n] = 0;
        }
        return;
    }
    const bool multi = C > 1;
    int bstar = -1;   // every visible pool is selected
    if (n_vis > select_k) {
        const uint4 *gh = reinterpret_cast<const uint4 *>(ghist + static_cast<int64_t>(n) * kHistBins);
        for (int i = tid; i < kHistBins / 4; i += blockDim.x) reinterpret_cast<uint4 *>(hist)[i] = __ldcg(gh + i);
        __syncthreads();
        block_find_bin(hist, static_cast<unsigned>(select_k), s);
        bstar = static_cast<int>(s.bin);
    }
    if (tid == 0) { s.n_a = 0; s.n_b = 0; }
    if (!multi)
        for (int i = tid; i < kHistBins; i += blockDim.x) s.hist2[i] = 0;
    __syncthreads();
    const int per = ((n_vis + C - 1) / C + 3) & ~3;
    const int lo = min(n_vis, c * per), hi = min(n_vis, lo + per);
    unsigned *h2 = multi ? ghist2 + static_cast<int64_t>(n) * kHistBins : s.hist2;
    auto score_at = [&](int i) { return __ldg(row + i); };
    classify_range(score_at, lo, hi, bstar, h2, s);
    __syncthreads();
    unsigned nA, nB;
    bool b_complete;
    if (multi) {
        if (!merge_lists_multi(counters + static_cast<int64_t>(n) * kCntWords, words + static_cast<int64_t>(n) * kMaxSelCtas,
                               alist + static_cast<int64_t>(n) * list_cap, blist + static_cast<int64_t>(n) * list_cap,
                               per, ghist2 + static_cast<int64_t>(n) * kHistBins, C, nA, nB, b_complete, s))
            return;
    } else {
        nA = min(s.n_a, static_cast<unsigned>(kMaxSelect));
        nB = s.n_b;
        b_complete = nB <= static_cast<unsigned>(kBoundCap);
    }
    const unsigned long long top = static_cast<unsigned long long>(bstar < 0 ? 0 : bstar);
    auto get_b = [&](int i) -> unsigned long long {   // list B straight from the scores
        const uint32_t key = score_key(__ldg(row + i));
        return (key >> (32 - kHistBitsTop)) == top ? compose(key, i) : 0ull;
    };
    finish_selection(count, nA, nB, b_complete, bstar, s.hist2, get_b, n_vis, s);
    write_selection(out, select_k, count, s);
    if (tid == 0 && n_sel_out) n_sel_out[n] = static_cast<int32_t>(count);
}

size_t topk_select_smem() { return sizeof(SelShared); }

// Zero the per-query histograms and counters of a selection (a kernel rather than a memset so
// that it chains with the neighbouring kernels under programmatic dependent launch).
__global__ void __launch_bounds__(256) zero_words_kernel(uint4 *__restrict__ p, int64_t n16) {
    pdl_begin();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

cudaError_t launch_zero(void *p, size_t bytes, cudaStream_t stream) {
    const int64_t n16 = static_cast<int64_t>((bytes + 15) / 16);
    if (n16 == 0) return cudaSuccess;
    int64_t blocks = (n16 + 255) / 256;
    if (blocks > 1184) blocks = 1184;
    launch_pdl(zero_words_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
               static_cast<uint4 *>(p), n16);
    return cudaGetLastError();
}
int topk_collect_ctas(int64_t ld) {
    int64_t c = ld / 2048;
    if (c < 1) c = 1;
    if (c > 64) c = 64;
    return static_cast<int>(c);
}

cudaError_t launch_topk_hist(const float *scores, const NvisSource &src, int n_q, unsigned *ghist,
                             cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>((src.ld + 8191) / 8192), n_q);
    if (grid.x == 0 || n_q == 0) return cudaSuccess;
    launch_pdl(topk_hist_kernel, dim3(grid), dim3(256), 0, stream, scores, src, ghist);
    return cudaGetLastError();
}

cudaError_t launch_topk_collect(const float *scores, const NvisSource &src, const unsigned *ghist,
                                unsigned *ghist2, unsigned *counters, unsigned *words, unsigned long long *alist,
                                unsigned long long *blist, int n_q, int select_k, int32_t *topk,
                                int32_t *n_sel, cudaStream_t stream) {
    const size_t smem = sizeof(SelShared);
    cudaError_t e = cudaFuncSetAttribute(topk_collect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(topk_collect_ctas(src.ld), n_q);
    launch_pdl(topk_collect_kernel, dim3(grid), dim3(kCollectThreads), smem, stream, scores, src, ghist, ghist2,
               counters, words, alist, blist, sel_list_cap(src.ld), select_k, topk, n_sel);
    return cudaGetLastError();
}

}  // namespace glm

namespace glm {

// Context parallelism (TensorFold issue #402, 'Credit': "local candidates are merged into the
// global top-k"): rank r of `world` holds the pools p = r + world i; its index kernel selected the
// select_k best of them by local index i. cp_candidates turns that selection into (score, global
// pool id) pairs; merge_topk selects the select_k best of every rank's pairs, by score descending
// and then the lower global id -- exactly the selection over all pools, because each pool of the
// global selection is among its own rank's select_k best.
__global__ void __launch_bounds__(256) cp_candidates_kernel(const float *__restrict__ scores, int64_t ld,
                                                            const int32_t *__restrict__ topk, int select_k,
                                                            int rank, int world, float *__restrict__ cand_scores,
                                                            int32_t *__restrict__ cand_ids) {
    pdl_begin();
    const int n = blockIdx.y;
    const int x = blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= select_k) return;
    const int64_t o = static_cast<int64_t>(n) * select_k + x;
    const int i = topk[o];
    const bool ok = i >= 0 && i < ld;
    cand_scores[o] = ok ? scores[static_cast<int64_t>(n) * ld + i] : 0.0f;
    cand_ids[o] = ok ? i * world + rank : GLM_INVALID;
}

// One CTA per query over the candidates of n_parts parts laid out [n_parts][n_q][per_part]
// (per_part = n_cand / n_parts): radix selection of the count best composites, bitonic sort,
// then the top-k row (-1 padded) and n_sel.
__global__ void __launch_bounds__(kCollectThreads) merge_topk_kernel(const float *__restrict__ cand_scores,
                                                                     const int32_t *__restrict__ cand_ids,
                                                                     int n_parts, int n_q, int per_part,
                                                                     int select_k, int32_t *__restrict__ topk,
                                                                     int32_t *__restrict__ n_sel) {
    pdl_begin();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SelShared &s = *reinterpret_cast<SelShared *>(smem_raw);
    const int n = blockIdx.x;
    const int m = n_parts * per_part;
    auto at = [&](int i) { return (static_cast<int64_t>(i / per_part) * n_q + n) * per_part + (i % per_part); };
    auto get = [&](int i) -> unsigned long long {
        const int32_t id = cand_ids[at(i)];
        return id >= 0 ? compose(score_key(cand_scores[at(i)]), id) : 0ull;
    };
    unsigned valid = 0u;
    for (int b0 = 0; b0 < m; b0 += blockDim.x) {
        const int i = b0 + static_cast<int>(threadIdx.x);
        valid += static_cast<unsigned>(__syncthreads_count(i < m && cand_ids[at(i)] >= 0));
    }
    const unsigned count = min(static_cast<unsigned>(select_k), valid);
    if (count > 0) {
        radix_select(get, m, count, 0, 0ull, s);
        collect_from(get, m, ~0ull << (64 - s.done), s.prefix, 0u, s);
        sort_selected(s.cand, static_cast<int>(count), s);
    }
    write_selection(topk + static_cast<int64_t>(n) * select_k, select_k, count, s);
    if (threadIdx.x == 0 && n_sel) n_sel[n] = static_cast<int32_t>(count);
}

cudaError_t launch_cp_candidates(const float *scores, int64_t ld, const int32_t *topk, int n_q, int select_k,
                                 int rank, int world, float *cand_scores, int32_t *cand_ids, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>((select_k + 255) / 256), static_cast<unsigned>(n_q));
    launch_pdl(cp_candidates_kernel, grid, dim3(256), 0, stream, scores, ld, topk, select_k, rank, world, cand_scores,
               cand_ids);
    return cudaGetLastError();
}

cudaError_t launch_merge_topk(const float *cand_scores, const int32_t *cand_ids, int n_parts, int n_q, int per_part,
                              int select_k, int32_t *topk, int32_t *n_sel, cudaStream_t stream) {
    const int smem = static_cast<int>(sizeof(SelShared));
    cudaError_t e = cudaFuncSetAttribute(merge_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    launch_pdl(merge_topk_kernel, dim3(static_cast<unsigned>(n_q)), dim3(kCollectThreads), smem, stream, cand_scores,
               cand_ids, n_parts, n_q, per_part, select_k, topk, n_sel);
    return cudaGetLastError();
}

}  // namespace glm
