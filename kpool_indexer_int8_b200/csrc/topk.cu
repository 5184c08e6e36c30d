// topk.cu -- selection of the select_k highest-scoring visible pools ("Module glm5next_dsa_ref",
// topk_pools), ordered by score descending with ties to the lower pool id.
//
// Keys: the fp32 score mapped to an order-preserving uint32 (-0.0 folded onto +0.0), extended to
// a unique 64-bit composite (key << 32 | ~pool_id) so that "larger composite" is exactly "higher
// score, then lower id".
//
//   1. histogram: a 2048-bin count of the top 11 key bits per query (built by the score kernel's
//      epilogue, or by topk_hist_kernel for caller-supplied scores);
//   2. select kernel, one CTA per query:
//        a. from the histogram, the bin b* holding the select_k-th largest key and the count of
//           keys in higher bins (always < select_k);
//        b. one pass over the scores keeps every key of a higher bin (list A) and every key of
//           bin b* (list B, in shared memory);
//        c. a radix select on the composites of B (8-bit digits over the remaining 53 bits,
//           stopping as soon as the digit holding the boundary is taken whole) picks the rest;
//        d. a bitonic sort of the select_k composites in shared memory gives the order.
//      If B exceeds its shared-memory capacity (massive ties at the boundary), step (c) runs the
//      same radix select over the scores in global memory instead.
#include "common.cuh"
#include "topk.cuh"

namespace glm {

constexpr int kSelThreads = 1024;
constexpr int kBoundCap = 8192;

__device__ __forceinline__ unsigned long long compose(uint32_t key, int id) {
    return (static_cast<unsigned long long>(key) << 32) |
           static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(id));
}

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
// histogram of caller-supplied scores: grid (chunks of 8192 scores, n_q), 256 threads
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_hist_kernel(const float *__restrict__ scores, NvisSource src,
                                                        unsigned *__restrict__ ghist) {
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
        uint32_t d = 0xffffffffu;
        if (i < n_vis) d = score_key(row[i]) >> (32 - kHistBitsTop);
        hist_add(hist, d);
    }
    __syncthreads();
    unsigned *g = ghist + static_cast<int64_t>(n) * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
        if (hist[i]) atomicAdd(&g[i], hist[i]);
}

// ------------------------------------------------------------------------------------------------
// select kernel
// ------------------------------------------------------------------------------------------------
struct SelSmem {
    unsigned long long cand[kMaxSelect];   // list A, then the final select_k composites
    unsigned long long bnd[kBoundCap];     // list B (keys of the boundary bin)
    unsigned hist[256];
    unsigned bin, above, n_a, n_b, done;
    unsigned long long prefix;
};

// On warp 0: in a histogram of `nbins` bins (a multiple of 32), the highest bin whose suffix count
// (that bin and all higher ones) reaches k; writes the bin, the count in higher bins and the
// bin's own count.
__device__ void find_bin_warp(const unsigned *hist, int nbins, unsigned k, unsigned *bin,
                              unsigned *above_out, unsigned *count_out) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;
    unsigned lane_sum = 0;
    for (int j = 0; j < per; j++) lane_sum += hist[per * lane + j];
    unsigned suf = lane_sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
    }
    unsigned above = suf - lane_sum;
    if (above < k && k <= suf) {
        for (int j = per - 1; j >= 0; j--) {
            const unsigned c = hist[per * lane + j];
            if (above + c >= k) {
                *bin = static_cast<unsigned>(per * lane + j);
                *above_out = above;
                if (count_out) *count_out = c;
                break;
            }
            above += c;
        }
    }
}

// Radix select of the k largest composites among the entries that share `prefix` on the bits of
// `mask` (known_bits leading bits). The entries come from `get(i)`, i < m. On return
// sm.prefix / sm.done describe the boundary: the selection is every entry e with
// (e & ~0 << (64 - done)) >= prefix, which holds exactly k entries.
template <typename Get>
__device__ void radix_select(Get get, int m, unsigned k, int known_bits, unsigned long long prefix,
                             SelSmem &sm) {
    const int tid = threadIdx.x;
    unsigned long long mask = ~0ull << (64 - known_bits);
    int bits = known_bits;
    while (bits < 64) {
        const int width = min(8, 64 - bits);
        const int shift = 64 - bits - width;
        for (int i = tid; i < 256; i += blockDim.x) sm.hist[i] = 0;
        if (tid == 0) { sm.bin = 0; sm.above = 0; sm.n_b = 0; }
        __syncthreads();
        for (int base = 0; base < m; base += blockDim.x) {
            const int i = base + tid;
            uint32_t d = 0xffffffffu;
            if (i < m) {
                unsigned long long c;
                if (get(i, c) && (c & mask) == prefix) d = static_cast<uint32_t>((c >> shift) & ((1u << width) - 1));
            }
            hist_add(sm.hist, d);
        }
        __syncthreads();
        if (tid < 32) find_bin_warp(sm.hist, 256, k, &sm.bin, &sm.above, &sm.n_b);
        __syncthreads();
        const unsigned d = sm.bin, above = sm.above, in_bin = sm.n_b;
        prefix |= static_cast<unsigned long long>(d) << shift;
        mask |= static_cast<unsigned long long>((1u << width) - 1) << shift;
        bits += width;
        k -= above;
        __syncthreads();
        if (k == in_bin) break;  // the whole digit is taken: resolved
    }
    if (tid == 0) { sm.prefix = prefix; sm.done = static_cast<unsigned>(bits); }
    __syncthreads();
}

__device__ void bitonic_desc(unsigned long long *a, int count) {
    int P2 = 1;
    while (P2 < count) P2 <<= 1;
    for (int i = count + threadIdx.x; i < P2; i += blockDim.x) a[i] = 0ull;
    __syncthreads();
    for (int k = 2; k <= P2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P2; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const unsigned long long x = a[i], y = a[ixj];
                    const bool desc = (i & k) == 0;
                    if (desc ? (x < y) : (x > y)) { a[i] = y; a[ixj] = x; }
                }
            }
            __syncthreads();
        }
    }
}

// Append every entry with get(i) valid and (c & msk) >= pre to sm.cand[base + ...].
template <typename Get>
__device__ void collect_from(Get get, int m, unsigned long long msk, unsigned long long pre,
                             unsigned base, SelSmem &sm) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) sm.n_b = 0;
    __syncthreads();
    for (int b0 = 0; b0 < m; b0 += blockDim.x) {
        const int i = b0 + threadIdx.x;
        unsigned long long c = 0;
        const bool take = i < m && get(i, c) && (c & msk) >= pre;
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        unsigned p = 0;
        if (lane == 0 && tm) p = atomicAdd(&sm.n_b, __popc(tm));
        p = __shfl_sync(0xffffffffu, p, 0);
        const unsigned pos = base + p + __popc(tm & ((1u << lane) - 1));
        if (take && pos < static_cast<unsigned>(kMaxSelect)) sm.cand[pos] = c;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(
    const float *__restrict__ scores, NvisSource src, const unsigned *__restrict__ ghist,
    int select_k, int32_t *__restrict__ topk, int32_t *__restrict__ n_sel_out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SelSmem &sm = *reinterpret_cast<SelSmem *>(smem_raw);
    const int n = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int n_vis = nvis_of(src, n);
    const float *row = scores + static_cast<int64_t>(n) * src.ld;
    int32_t *out = topk + static_cast<int64_t>(n) * select_k;
    const int n_sel = min(select_k, n_vis);
    int count;
    if (n_vis <= select_k) {
        for (int i = tid; i < n_vis; i += blockDim.x) sm.cand[i] = compose(score_key(row[i]), i);
        count = n_vis;
        __syncthreads();
    } else {
        // (a) the boundary bin from the 2048-bin histogram (defaults keep every write in bounds
        // should the histogram not match the scores)
        if (tid == 0) { sm.bin = 0; sm.above = 0; sm.n_b = 0xffffffffu; }
        unsigned *h_stage = reinterpret_cast<unsigned *>(sm.bnd);  // free until step (b)
        for (int i = tid; i < kHistBins; i += blockDim.x) h_stage[i] = ghist[static_cast<int64_t>(n) * kHistBins + i];
        __syncthreads();
        if (tid < 32) find_bin_warp(h_stage, kHistBins, static_cast<unsigned>(select_k), &sm.bin, &sm.above, &sm.n_b);
        if (tid == 0) sm.n_a = 0;
        __syncthreads();
        const unsigned bstar = sm.bin, n_above = sm.above, m_b = sm.n_b;
        const bool fits = m_b <= static_cast<unsigned>(kBoundCap);
        __syncthreads();
        if (tid == 0) sm.n_b = 0;
        __syncthreads();
        // (b) one pass: A = keys of higher bins, B = keys of the boundary bin. 16 scores per thread
        // per round (four 16-byte loads when the row is 16-byte aligned) keep ~64 KB in flight.
        auto classify = [&](int idx, uint32_t key, bool ok) {
            const unsigned d = key >> (32 - kHistBitsTop);
            const bool a = ok && d > bstar;
            const bool bb = ok && fits && d == bstar;
            const unsigned am = __ballot_sync(0xffffffffu, a);
            const unsigned bm = __ballot_sync(0xffffffffu, bb);
            unsigned pa = 0, pb = 0;
            if (lane == 0) {
                if (am) pa = atomicAdd(&sm.n_a, __popc(am));
                if (bm) pb = atomicAdd(&sm.n_b, __popc(bm));
            }
            pa = __shfl_sync(0xffffffffu, pa, 0);
            pb = __shfl_sync(0xffffffffu, pb, 0);
            const unsigned lt = (1u << lane) - 1;
            const unsigned ra = pa + __popc(am & lt), rb = pb + __popc(bm & lt);
            if (a && ra < static_cast<unsigned>(kMaxSelect)) sm.cand[ra] = compose(key, idx);
            if (bb && rb < static_cast<unsigned>(kBoundCap)) sm.bnd[rb] = compose(key, idx);
        };
        if ((reinterpret_cast<uintptr_t>(row) & 15) == 0) {
            const int n4 = n_vis >> 2;
            const float4 *row4 = reinterpret_cast<const float4 *>(row);
            for (int base = 0; base < n4; base += blockDim.x * 4) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int i4 = base + u * blockDim.x + tid;
                    v[u] = i4 < n4 ? row4[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int i4 = base + u * blockDim.x + tid;
                    const bool ok = i4 < n4;
                    classify(4 * i4 + 0, score_key(v[u].x), ok);
                    classify(4 * i4 + 1, score_key(v[u].y), ok);
                    classify(4 * i4 + 2, score_key(v[u].z), ok);
                    classify(4 * i4 + 3, score_key(v[u].w), ok);
                }
            }
            for (int i = 4 * n4 + tid; i < 4 * n4 + 32 * ((n_vis - 4 * n4 + 31) / 32); i += blockDim.x)
                classify(i, i < n_vis ? score_key(row[i]) : 0u, i < n_vis);
        } else {
            for (int base = 0; base < n_vis; base += blockDim.x * 4) {
                uint32_t key[4];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int i = base + u * blockDim.x + tid;
                    key[u] = i < n_vis ? score_key(row[i]) : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int i = base + u * blockDim.x + tid;
                    classify(i, key[u], i < n_vis);
                }
            }
        }
        __syncthreads();
        // (c) the remaining select_k - n_above keys from the boundary bin
        const unsigned need = static_cast<unsigned>(select_k) - min(n_above, static_cast<unsigned>(select_k));
        const unsigned long long top = static_cast<unsigned long long>(bstar) << (64 - kHistBitsTop);
        if (fits) {
            const int m = static_cast<int>(min(sm.n_b, static_cast<unsigned>(kBoundCap)));
            auto get = [&](int i, unsigned long long &c) { c = sm.bnd[i]; return true; };
            if (static_cast<unsigned>(m) == need) {
                for (int i = tid; i < m; i += blockDim.x)
                    if (n_above + i < static_cast<unsigned>(kMaxSelect)) sm.cand[n_above + i] = sm.bnd[i];
                __syncthreads();
            } else {
                radix_select(get, m, need, kHistBitsTop, top, sm);
                collect_from(get, m, ~0ull << (64 - sm.done), sm.prefix, n_above, sm);
            }
        } else {
            auto get = [&](int i, unsigned long long &c) {
                const uint32_t key = score_key(row[i]);
                c = compose(key, i);
                return (key >> (32 - kHistBitsTop)) == bstar;
            };
            radix_select(get, n_vis, need, kHistBitsTop, top, sm);
            collect_from(get, n_vis, ~0ull << (64 - sm.done), sm.prefix, n_above, sm);
        }
        count = select_k;
    }
    // (d) order
    bitonic_desc(sm.cand, count);
    for (int i = tid; i < select_k; i += blockDim.x)
        out[i] = i < n_sel ? static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(sm.cand[i] & 0xffffffffu))
                           : GLM_INVALID;
    if (tid == 0 && n_sel_out) n_sel_out[n] = n_sel;
}

size_t topk_select_smem() { return sizeof(SelSmem); }

cudaError_t launch_topk_hist(const float *scores, const NvisSource &src, int n_q, unsigned *ghist,
                             cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>((src.ld + 8191) / 8192), n_q);
    if (grid.x == 0 || n_q == 0) return cudaSuccess;
    topk_hist_kernel<<<grid, 256, 0, stream>>>(scores, src, ghist);
    return cudaGetLastError();
}

cudaError_t launch_topk_select(const float *scores, const NvisSource &src, const unsigned *ghist,
                               int n_q, int select_k, int32_t *topk, int32_t *n_sel,
                               cudaStream_t stream) {
    const size_t smem = sizeof(SelSmem);
    cudaError_t e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    topk_select_kernel<<<n_q, kSelThreads, smem, stream>>>(scores, src, ghist, select_k, topk, n_sel);
    return cudaGetLastError();
}

}  // namespace glm
