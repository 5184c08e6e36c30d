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

constexpr int kCollectThreads = 1024;
constexpr int kBoundCap = 4096;

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

// Block-wide version for a 2048-bin histogram in shared memory (blockDim.x >= 256): each of the
// first 256 threads sums 8 contiguous bins (two 16-byte reads, conflict-free), warp 0 searches the
// 256 partial sums with find_bin_warp and then the 8 bins of the partial it lands in. Every
// thread must call it; the result is in sm.bin / sm.above / sm.n_b after the call.
__device__ void find_bin_block2048(const unsigned *hist, unsigned k, unsigned *partial, SelSmem &sm) {
    const int t = threadIdx.x;
    if (t < 256) {
        const uint4 a = reinterpret_cast<const uint4 *>(hist)[2 * t];
        const uint4 b = reinterpret_cast<const uint4 *>(hist)[2 * t + 1];
        partial[t] = (a.x + a.y) + (a.z + a.w) + (b.x + b.y) + (b.z + b.w);
    }
    __syncthreads();
    if (t < 32) {
        unsigned pbin = 0, pabove = 0, pcount = 0;
        find_bin_warp(partial, 256, k, &sm.bin, &sm.above, &sm.n_b);
        __syncwarp();
        if (t == 0) {
            pbin = sm.bin;
            pabove = sm.above;
            (void)pcount;
            unsigned above = pabove;
            for (int j = 7; j >= 0; j--) {   // the 8 bins of that partial, highest first
                const unsigned c = hist[8 * pbin + j];
                if (above + c >= k) {
                    sm.bin = 8 * pbin + j;
                    sm.above = above;
                    sm.n_b = c;
                    break;
                }
                above += c;
            }
        }
    }
    __syncthreads();
}

// Radix select of the k largest composites among the entries that share `prefix` on the bits of
// `mask` (known_bits leading bits). Entry i < m is get(i); 0 means "no entry" (a composite of a
// real score is never 0). On return sm.prefix / sm.done describe the boundary: the selection is
// every entry e with (e & ~0 << (64 - done)) >= prefix, which holds exactly k entries.
template <typename Get>
__device__ __forceinline__ void radix_select(const Get &get, int m, unsigned k, int known_bits,
                                             unsigned long long prefix, SelSmem &sm) {
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
                const unsigned long long c = get(i);
                if (c != 0ull && (c & mask) == prefix) d = static_cast<uint32_t>((c >> shift) & ((1u << width) - 1));
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

// Append every entry with get(i) != 0 and (c & msk) >= pre to sm.cand[base + ...].
template <typename Get>
__device__ __forceinline__ void collect_from(const Get &get, int m, unsigned long long msk,
                                             unsigned long long pre, unsigned base, SelSmem &sm) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) sm.n_b = 0;
    __syncthreads();
    for (int b0 = 0; b0 < m; b0 += blockDim.x) {
        const int i = b0 + threadIdx.x;
        const unsigned long long c = i < m ? get(i) : 0ull;
        const bool take = c != 0ull && (c & msk) >= pre;
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        unsigned p = 0;
        if (lane == 0 && tm) p = atomicAdd(&sm.n_b, __popc(tm));
        p = __shfl_sync(0xffffffffu, p, 0);
        const unsigned pos = base + p + __popc(tm & ((1u << lane) - 1));
        if (take && pos < static_cast<unsigned>(kMaxSelect)) sm.cand[pos] = c;
    }
    __syncthreads();
}

// Sort of up to kMaxSelect unique composites, descending: each warp sorts runs of 64 in registers
// (bitonic network over shuffles, two elements per lane), then every element's final position is
// its index in its run plus, for every other run, the number of entries greater than it (binary
// search). Writes row[pos] = pool id for pos < n_sel and -1 for n_sel <= pos < select_k.
__device__ __forceinline__ unsigned long long cmpx(unsigned long long mine, unsigned long long other, bool keep_max) {
    return keep_max ? (mine > other ? mine : other) : (mine < other ? mine : other);
}

__device__ void sort_and_write(unsigned long long *a, int count, int n_sel, int select_k, int32_t *__restrict__ row) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int runs = (count + 63) >> 6;
    for (int i = count + tid; i < runs * 64; i += blockDim.x) a[i] = 0ull;   // 0 sorts last
    __syncthreads();
    for (int r = warp; r < runs; r += nw) {
        unsigned long long e0 = a[64 * r + lane], e1 = a[64 * r + 32 + lane];
#pragma unroll
        for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
            for (int j = k >> 1; j > 0; j >>= 1) {
                if (j == 32) {          // partners are the two registers of one lane (k == 64)
                    const unsigned long long hi = e0 > e1 ? e0 : e1, lo = e0 > e1 ? e1 : e0;
                    e0 = hi;
                    e1 = lo;
                } else {
                    const unsigned long long o0 = __shfl_xor_sync(0xffffffffu, e0, j);
                    const unsigned long long o1 = __shfl_xor_sync(0xffffffffu, e1, j);
                    const int p0 = lane, p1 = lane + 32;
                    e0 = cmpx(e0, o0, ((p0 & k) == 0) == ((p0 & j) == 0));
                    e1 = cmpx(e1, o1, ((p1 & k) == 0) == ((p1 & j) == 0));
                }
            }
        }
        a[64 * r + lane] = e0;
        a[64 * r + 32 + lane] = e1;
    }
    __syncthreads();
    for (int i = tid; i < runs * 64; i += blockDim.x) {
        const unsigned long long x = a[i];
        const int r = i >> 6;
        int pos = i & 63;
        for (int q = 0; q < runs; q++) {
            if (q == r) continue;
            const unsigned long long *run = a + 64 * q;
            int lo = 0;                                    // entries of run q greater than x
#pragma unroll
            for (int step = 32; step > 0; step >>= 1)
                if (run[lo + step - 1] > x) lo += step;
            if (run[63] > x) lo = 64;
            pos += lo;
        }
        if (x != 0ull && pos < n_sel)
            row[pos] = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(x & 0xffffffffu));
    }
    for (int i = n_sel + tid; i < select_k; i += blockDim.x) row[i] = GLM_INVALID;
}

// grid (C, n_q), kCollectThreads threads. Every CTA of a query scans a slice of its scores, keeps
// the keys above the boundary bin (list A) and of the boundary bin (list B) in shared memory and
// appends them to the query's global lists with one atomic per list; the last CTA to finish
// (ticket) finishes the selection and writes the row.
__global__ void __launch_bounds__(kCollectThreads) topk_collect_kernel(
    const float *__restrict__ scores, NvisSource src, const unsigned *__restrict__ ghist,
    unsigned *__restrict__ counters, unsigned long long *__restrict__ alist,
    unsigned long long *__restrict__ blist, int64_t blist_ld, int select_k,
    int32_t *__restrict__ topk, int32_t *__restrict__ n_sel_out) {
    pdl_begin();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SelSmem &sm = *reinterpret_cast<SelSmem *>(smem_raw);
    __shared__ __align__(16) unsigned h_stage[kHistBins];
    __shared__ unsigned partial[256];
    __shared__ unsigned s_last, s_na, s_nb, s_base_a, s_base_b;
    const int n = blockIdx.y, c = blockIdx.x, C = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int n_vis = nvis_of(src, n);
    const float *row = scores + static_cast<int64_t>(n) * src.ld;
    int32_t *out = topk + static_cast<int64_t>(n) * select_k;
    const int n_sel = min(select_k, n_vis);
    if (n_vis <= select_k) {  // every visible pool is selected: CTA 0 sorts them
        if (c != 0) return;
        for (int i = tid; i < n_vis; i += blockDim.x) sm.cand[i] = compose(score_key(row[i]), i);
        __syncthreads();
        sort_and_write(sm.cand, n_vis, n_sel, select_k, out);
        if (tid == 0 && n_sel_out) n_sel_out[n] = n_sel;
        return;
    }
    unsigned *cnt = counters + 4 * static_cast<int64_t>(n);   // [A count, B count, tickets, -]
    unsigned long long *al = alist + static_cast<int64_t>(n) * kMaxSelect;
    unsigned long long *bl = blist + static_cast<int64_t>(n) * blist_ld;

    // (a) the boundary bin from the histogram
    if (tid == 0) { sm.bin = 0; sm.above = 0; sm.n_b = 0; s_na = 0; s_nb = 0; }
    {   // all loads first: one round trip
        static_assert(kHistBins % kCollectThreads == 0, "histogram staging");
        unsigned hv[kHistBins / kCollectThreads];
#pragma unroll
        for (int u = 0; u < kHistBins / kCollectThreads; u++)
            hv[u] = __ldcg(&ghist[static_cast<int64_t>(n) * kHistBins + u * kCollectThreads + tid]);
#pragma unroll
        for (int u = 0; u < kHistBins / kCollectThreads; u++) h_stage[u * kCollectThreads + tid] = hv[u];
    }
    __syncthreads();
    find_bin_block2048(h_stage, static_cast<unsigned>(select_k), partial, sm);
    const unsigned bstar = sm.bin, n_above = min(sm.above, static_cast<unsigned>(select_k - 1));

    // (b) this CTA's slice into local lists (A: sm.cand, B: sm.bnd), shared-memory atomics only
    const int per = ((n_vis + C - 1) / C + 3) & ~3;
    const int lo = min(n_vis, c * per), hi = min(n_vis, lo + per);
    auto classify = [&](int idx, uint32_t key, bool ok) {
        const unsigned d = key >> (32 - kHistBitsTop);
        const bool a = ok && d > bstar;
        const bool bb = ok && d == bstar;
        if (!__any_sync(0xffffffffu, a || bb)) return;
        const unsigned am = __ballot_sync(0xffffffffu, a);
        const unsigned bm = __ballot_sync(0xffffffffu, bb);
        unsigned pa = 0, pb = 0;
        if (lane == 0) {
            if (am) pa = atomicAdd(&s_na, __popc(am));
            if (bm) pb = atomicAdd(&s_nb, __popc(bm));
        }
        pa = __shfl_sync(0xffffffffu, pa, 0);
        pb = __shfl_sync(0xffffffffu, pb, 0);
        const unsigned lt = (1u << lane) - 1;
        const unsigned ra = pa + __popc(am & lt), rb = pb + __popc(bm & lt);
        if (a && ra < static_cast<unsigned>(kMaxSelect)) sm.cand[ra] = compose(key, idx);
        if (bb && rb < static_cast<unsigned>(kBoundCap)) sm.bnd[rb] = compose(key, idx);
    };
    const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15) == 0);
    if (vec) {
        const float4 *row4 = reinterpret_cast<const float4 *>(row);
        const int lo4 = lo >> 2, hi4 = hi >> 2;   // lo is a multiple of 4
        for (int base = lo4; base < hi4; base += blockDim.x * 2) {
            float4 v[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i4 = base + u * blockDim.x + tid;
                v[u] = i4 < hi4 ? __ldcg(row4 + i4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i4 = base + u * blockDim.x + tid;
                const bool ok = i4 < hi4;
                classify(4 * i4 + 0, score_key(v[u].x), ok);
                classify(4 * i4 + 1, score_key(v[u].y), ok);
                classify(4 * i4 + 2, score_key(v[u].z), ok);
                classify(4 * i4 + 3, score_key(v[u].w), ok);
            }
        }
        if (tid < 32) {  // at most 3 scores past the last full vector
            const int i = 4 * hi4 + tid;
            classify(i, i < hi ? score_key(row[i]) : 0u, i < hi);
        }
    } else {
        for (int base = lo; base < hi; base += blockDim.x) {
            const int i = base + tid;
            classify(i, i < hi ? score_key(row[i]) : 0u, i < hi);
        }
    }
    __syncthreads();
    const unsigned la = min(s_na, static_cast<unsigned>(kMaxSelect)), lb = min(s_nb, static_cast<unsigned>(kBoundCap));
    if (tid == 0) {
        s_base_a = la ? atomicAdd(&cnt[0], la) : 0u;
        s_base_b = lb ? atomicAdd(&cnt[1], lb) : 0u;
    }
    __syncthreads();
    for (unsigned i = tid; i < la; i += blockDim.x)
        if (s_base_a + i < static_cast<unsigned>(kMaxSelect)) al[s_base_a + i] = sm.cand[i];
    for (unsigned i = tid; i < lb; i += blockDim.x)
        if (s_base_b + i < static_cast<unsigned long long>(blist_ld)) bl[s_base_b + i] = sm.bnd[i];

    // (c) the last CTA of the query finishes the selection and writes the row
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&cnt[2], 1u) == static_cast<unsigned>(C - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const unsigned nA = min(__ldcg(&cnt[0]), n_above);
    const unsigned nB = min(static_cast<unsigned long long>(__ldcg(&cnt[1])), static_cast<unsigned long long>(blist_ld));
    const unsigned need = static_cast<unsigned>(select_k) - nA;
    const bool b_fits = nB <= static_cast<unsigned>(kBoundCap);
    for (unsigned i0 = 0; i0 < nA + (b_fits ? nB : 0u); i0 += 8 * blockDim.x) {
        unsigned long long v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const unsigned i = i0 + u * blockDim.x + tid;
            v[u] = i < nA ? __ldcg(&al[i]) : (i < nA + nB ? __ldcg(&bl[i - nA]) : 0ull);
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const unsigned i = i0 + u * blockDim.x + tid;
            if (i < nA) sm.cand[i] = v[u];
            else if (b_fits && i < nA + nB) sm.bnd[i - nA] = v[u];
        }
    }
    __syncthreads();
    if (b_fits && nB == need) {
        for (unsigned i = tid; i < nB; i += blockDim.x)
            if (nA + i < static_cast<unsigned>(kMaxSelect)) sm.cand[nA + i] = sm.bnd[i];
        __syncthreads();
    } else if (b_fits) {
        // one more 11-bit level over list B (composite bits 52..42), in shared memory
        constexpr int kShift2 = 64 - 2 * kHistBitsTop;
        for (int i = tid; i < kHistBins; i += blockDim.x) h_stage[i] = 0;
        if (tid == 0) { sm.bin = 0; sm.above = 0; sm.n_b = 0; s_na = 0; s_nb = 0; }
        __syncthreads();
        for (unsigned base = 0; base < nB; base += blockDim.x) {
            const unsigned i = base + tid;
            const uint32_t d = i < nB ? static_cast<uint32_t>((sm.bnd[i] >> kShift2) & (kHistBins - 1)) : 0xffffffffu;
            hist_add(h_stage, d);
        }
        __syncthreads();
        find_bin_block2048(h_stage, need, partial, sm);
        const unsigned b2 = sm.bin, above2 = min(sm.above, need - 1), m2 = sm.n_b;
        // entries above the sub-bin are selected; the sub-bin's entries go to a short list
        constexpr int kSub = 256;
        unsigned long long *sub = reinterpret_cast<unsigned long long *>(h_stage);   // 2048 x 4 B = 256 x 8 B
        const bool small = m2 <= static_cast<unsigned>(kSub);
        __syncthreads();
        for (unsigned base = 0; base < nB; base += blockDim.x) {
            const unsigned i = base + tid;
            const unsigned long long x = i < nB ? sm.bnd[i] : 0ull;
            const unsigned d = static_cast<unsigned>((x >> kShift2) & (kHistBins - 1));
            const bool up = i < nB && d > b2;
            const bool eq = small && i < nB && d == b2;
            const unsigned um = __ballot_sync(0xffffffffu, up), em = __ballot_sync(0xffffffffu, eq);
            unsigned pu = 0, pe = 0;
            if (lane == 0) {
                if (um) pu = atomicAdd(&s_na, __popc(um));
                if (em) pe = atomicAdd(&s_nb, __popc(em));
            }
            pu = __shfl_sync(0xffffffffu, pu, 0);
            pe = __shfl_sync(0xffffffffu, pe, 0);
            const unsigned lt = (1u << lane) - 1;
            const unsigned ru = nA + pu + __popc(um & lt), re = pe + __popc(em & lt);
            if (up && ru < static_cast<unsigned>(kMaxSelect)) sm.cand[ru] = x;
            if (eq && re < static_cast<unsigned>(kSub)) sub[re] = x;
        }
        __syncthreads();
        (void)above2;
        const unsigned need2 = need - min(s_na, need);   // still needed from the sub-bin
        if (small) {
            // rank inside the sub-bin (unique composites): keep the need2 largest
            const unsigned base2 = nA + s_na;
            for (unsigned i = tid; i < m2; i += blockDim.x) {
                const unsigned long long x = sub[i];
                unsigned rank = 0;
                for (unsigned j = 0; j < m2; j++) rank += sub[j] > x;
                if (rank < need2 && base2 + rank < static_cast<unsigned>(kMaxSelect)) sm.cand[base2 + rank] = x;
            }
            __syncthreads();
        } else {  // a large sub-bin (ties at the boundary): the general radix selection over B
            auto get = [&](int i) { return sm.bnd[i]; };
            const unsigned long long top = static_cast<unsigned long long>(bstar) << (64 - kHistBitsTop);
            radix_select(get, static_cast<int>(nB), need, kHistBitsTop, top, sm);
            collect_from(get, static_cast<int>(nB), ~0ull << (64 - sm.done), sm.prefix, nA, sm);
        }
    } else {  // a very large boundary bin (massive ties): select straight from the global list
        auto get = [&](int i) { return __ldcg(&bl[i]); };
        const unsigned long long top = static_cast<unsigned long long>(bstar) << (64 - kHistBitsTop);
        radix_select(get, static_cast<int>(nB), need, kHistBitsTop, top, sm);
        collect_from(get, static_cast<int>(nB), ~0ull << (64 - sm.done), sm.prefix, nA, sm);
    }
    sort_and_write(sm.cand, select_k, n_sel, select_k, out);
    if (tid == 0 && n_sel_out) n_sel_out[n] = n_sel;
}

size_t topk_select_smem() { return sizeof(SelSmem); }

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
                                unsigned *counters, unsigned long long *alist,
                                unsigned long long *blist, int n_q, int select_k, int32_t *topk,
                                int32_t *n_sel, cudaStream_t stream) {
    const size_t smem = sizeof(SelSmem);
    cudaError_t e = cudaFuncSetAttribute(topk_collect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const long long blist_ld = src.ld > 0 ? src.ld : 1;
    dim3 grid(topk_collect_ctas(src.ld), n_q);
    launch_pdl(topk_collect_kernel, dim3(grid), dim3(kCollectThreads), smem, stream, scores, src, ghist, counters, alist, blist,
                                                                blist_ld, select_k, topk, n_sel);
    return cudaGetLastError();
}

}  // namespace glm
