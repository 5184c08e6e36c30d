// topk.cu -- selection of the select_k highest-scoring visible pools ("Module glm5next_dsa_ref",
// topk_pools), ordered by score descending with ties to the lower pool id.
//
// One CTA of 1024 threads per query:
//   1. radix select (four 8-bit digits, most significant first) of the select_k-th largest
//      32-bit order-preserving score key T, with warp-aggregated shared-memory histograms;
//   2. one ordered pass that keeps every key > T and the lowest-id keys == T (a block-wide
//      prefix count in pool-id order decides which of the equal keys are taken);
//   3. a bitonic sort of the kept (key, ~id) 64-bit composites in shared memory.
// When n_vis <= select_k every visible pool is kept and only step 3 runs.
#include "common.cuh"

namespace glm {

constexpr int kTopkThreads = 1024;

struct TopkSmem {
    unsigned long long cand[kMaxSelect];
    unsigned int hist[256];
    unsigned int warp_tot[32];
    unsigned int prefix, k_rem, n_gt, eq_base;
};

__device__ __forceinline__ unsigned long long compose(uint32_t key, int id) {
    return (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(id));
}

// Select and sort for one query; `scores` holds n_vis valid entries.
__device__ void topk_block(const float *__restrict__ scores, int n_vis, int select_k,
                           int32_t *__restrict__ topk_out, int32_t *__restrict__ n_sel_out,
                           TopkSmem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_sel = min(select_k, n_vis);
    int count;
    if (n_vis <= select_k) {
        for (int i = tid; i < n_vis; i += blockDim.x) sm.cand[i] = compose(score_key(scores[i]), i);
        count = n_vis;
    } else {
        if (tid == 0) { sm.prefix = 0; sm.k_rem = select_k; }
        uint32_t mask = 0;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += blockDim.x) sm.hist[i] = 0;
            __syncthreads();
            const uint32_t prefix = sm.prefix;
            for (int base = 0; base < n_vis; base += blockDim.x) {
                const int i = base + tid;
                uint32_t digit = 0xffffffffu;
                if (i < n_vis) {
                    const uint32_t key = score_key(scores[i]);
                    if ((key & mask) == prefix) digit = (key >> shift) & 0xffu;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, digit);
                if (digit != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[digit], __popc(peers));
            }
            __syncthreads();
            if (warp == 0) {
                // lane l owns digits [8l, 8l + 8); find the digit holding the k_rem-th largest
                unsigned cnt[8], lane_sum = 0;
#pragma unroll
                for (int j = 0; j < 8; j++) { cnt[j] = sm.hist[8 * lane + j]; lane_sum += cnt[j]; }
                unsigned suf = lane_sum;  // inclusive suffix sum over lanes >= lane
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    unsigned v = __shfl_down_sync(0xffffffffu, suf, o);
                    if (lane + o < 32) suf += v;
                }
                unsigned above = suf - lane_sum;
                const unsigned k = sm.k_rem;
                if (above < k && k <= suf) {
                    for (int j = 7; j >= 0; j--) {
                        if (above + cnt[j] >= k) {
                            sm.prefix = prefix | (static_cast<uint32_t>(8 * lane + j) << shift);
                            sm.k_rem = k - above;
                            break;
                        }
                        above += cnt[j];
                    }
                }
            }
            mask |= 0xffu << shift;
            __syncthreads();
        }
        const uint32_t T = sm.prefix;
        const unsigned need_eq = sm.k_rem;
        const unsigned n_gt = static_cast<unsigned>(select_k) - need_eq;
        if (tid == 0) { sm.n_gt = 0; sm.eq_base = 0; }
        __syncthreads();
        for (int base = 0; base < n_vis; base += blockDim.x) {
            const int i = base + tid;
            uint32_t key = 0;
            if (i < n_vis) key = score_key(scores[i]);
            const bool gt = i < n_vis && key > T;
            const bool eq = i < n_vis && key == T;
            const unsigned gt_mask = __ballot_sync(0xffffffffu, gt);
            unsigned gpos = 0;
            if (lane == 0 && gt_mask) gpos = atomicAdd(&sm.n_gt, __popc(gt_mask));
            gpos = __shfl_sync(0xffffffffu, gpos, 0);
            if (gt) sm.cand[gpos + __popc(gt_mask & ((1u << lane) - 1))] = compose(key, i);
            const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
            if (lane == 0) sm.warp_tot[warp] = __popc(eq_mask);
            __syncthreads();
            if (eq) {
                unsigned off = sm.eq_base;
                for (int w = 0; w < warp; w++) off += sm.warp_tot[w];
                const unsigned rank = off + __popc(eq_mask & ((1u << lane) - 1));
                if (rank < need_eq) sm.cand[n_gt + rank] = compose(key, i);
            }
            __syncthreads();
            if (tid == 0) {
                unsigned tot = 0;
                for (int w = 0; w < (blockDim.x >> 5); w++) tot += sm.warp_tot[w];
                sm.eq_base += tot;
            }
            __syncthreads();
        }
        count = select_k;
    }
    // bitonic sort of cand[0, P2) descending; padding zeros sort last
    int P2 = 1;
    while (P2 < count) P2 <<= 1;
    for (int i = count + tid; i < P2; i += blockDim.x) sm.cand[i] = 0ull;
    __syncthreads();
    for (int k = 2; k <= P2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P2; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const unsigned long long a = sm.cand[i], b = sm.cand[ixj];
                    const bool desc = (i & k) == 0;
                    if (desc ? (a < b) : (a > b)) { sm.cand[i] = b; sm.cand[ixj] = a; }
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < select_k; i += blockDim.x)
        topk_out[i] = i < n_sel ? static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(sm.cand[i] & 0xffffffffu)) : GLM_INVALID;
    if (tid == 0 && n_sel_out) *n_sel_out = n_sel;
}

// Selection for the fused entry: n_vis from the query's sequence geometry.
__global__ void __launch_bounds__(kTopkThreads) topk_fused_kernel(
    const float *__restrict__ scores, int64_t ld_scores, const int32_t *__restrict__ q_seq,
    const int32_t *__restrict__ q_pos, const int32_t *__restrict__ pad,
    const int32_t *__restrict__ len, int batch, int select_k, int32_t *__restrict__ topk,
    int32_t *__restrict__ n_sel) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    const int n = blockIdx.x;
    const int b = q_seq[n];
    const int n_vis = (b >= 0 && b < batch) ? visible_pools(pad[b], len[b], q_pos[n], ld_scores) : 0;
    topk_block(scores + static_cast<int64_t>(n) * ld_scores, n_vis, select_k,
               topk + static_cast<int64_t>(n) * select_k, n_sel ? n_sel + n : nullptr, sm);
}

// Selection on caller-supplied scores: n_vis given per query.
__global__ void __launch_bounds__(kTopkThreads) topk_given_kernel(
    const float *__restrict__ scores, int64_t ld_scores, const int32_t *__restrict__ n_visible,
    int select_k, int32_t *__restrict__ topk, int32_t *__restrict__ n_sel) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    const int n = blockIdx.x;
    long long nv = n_visible[n];
    if (nv < 0) nv = 0;
    if (nv > ld_scores) nv = ld_scores;
    const int n_vis = static_cast<int>(nv);
    topk_block(scores + static_cast<int64_t>(n) * ld_scores, n_vis, select_k,
               topk + static_cast<int64_t>(n) * select_k, n_sel ? n_sel + n : nullptr, sm);
}

cudaError_t launch_topk_fused(const float *scores, int64_t ld_scores, const int32_t *q_seq,
                              const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                              int batch, int n_q, int select_k, int32_t *topk, int32_t *n_sel,
                              cudaStream_t stream) {
    const size_t smem = sizeof(TopkSmem);
    cudaError_t e = cudaFuncSetAttribute(topk_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    topk_fused_kernel<<<n_q, kTopkThreads, smem, stream>>>(scores, ld_scores, q_seq, q_pos, pad,
                                                           len, batch, select_k, topk, n_sel);
    return cudaGetLastError();
}

cudaError_t launch_topk_given(const float *scores, int64_t ld_scores, const int32_t *n_visible,
                              int n_q, int select_k, int32_t *topk, int32_t *n_sel,
                              cudaStream_t stream) {
    const size_t smem = sizeof(TopkSmem);
    cudaError_t e = cudaFuncSetAttribute(topk_given_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    topk_given_kernel<<<n_q, kTopkThreads, smem, stream>>>(scores, ld_scores, n_visible, select_k,
                                                           topk, n_sel);
    return cudaGetLastError();
}

}  // namespace glm
