// select.cuh -- block-level pieces of the top-k pool selection ("Module glm5next_dsa_ref",
// topk_pools: the select_k highest scores, by score descending, ties to the lower pool id),
// shared by the fused score+select kernel and the selection kernel on given scores.
//
// Keys: the fp32 score mapped to an order-preserving uint32 (-0.0 folded onto +0.0), extended to
// a unique 64-bit composite (key << 32 | ~pool_id), so that "larger composite" is exactly "higher
// score, then lower id". The selection never compares floats.
//
//   level 1: a 2048-bin histogram of the top 11 key bits gives the boundary bin b* (the bin of
//            the select_k-th largest key) and the count above it; keys above b* form list A
//            (always fewer than select_k), keys in b* form list B;
//   level 2: a 2048-bin histogram of the next 11 bits over list B gives the boundary sub-bin;
//            keys above it are taken, the few keys of the sub-bin are ranked directly;
//   fallback: a radix selection over the composites (8-bit digits) when the sub-bin is large or
//            list B did not fit on chip (massive ties);
//   order:    a bucketed counting sort of the selected composites, descending (a bitonic sort
//             when the composites cluster in few buckets).
// Histograms use plain shared-memory atomics: warp match instructions are far slower here.
#pragma once

#include "common.cuh"
#include "topk.cuh"

namespace glm {

constexpr int kBoundCap = 4096;                  // list B entries kept on chip
constexpr int kSubCap = 256;                     // level-2 boundary entries ranked directly
constexpr int kShift2 = 64 - 2 * kHistBitsTop;   // level-2 digit: composite bits 52..42
constexpr uint32_t kSelWaitLimit = 1u << 21;     // polls of a cross-CTA wait before giving up
// The limit the waits use: kSelWaitLimit unless a test lowers it (glm_debug_set_cross_cta_wait_limit)
// to make a wait run out on purpose. One copy per translation unit that waits across CTAs.
static __device__ uint32_t g_cross_cta_wait_limit = kSelWaitLimit;

__device__ __forceinline__ unsigned long long compose(uint32_t key, int id) {
    return (static_cast<unsigned long long>(key) << 32) |
           static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(id));
}
__device__ __forceinline__ int id_of(unsigned long long c) {
    return static_cast<int>(0xffffffffu - static_cast<uint32_t>(c & 0xffffffffu));
}

// Working set of one CTA's selection (overlaid on memory the scoring no longer needs).
struct SelShared {
    unsigned long long cand[kMaxSelect];   // list A, then the whole selection (sorted in place)
    unsigned long long bnd[kBoundCap];     // list B
    unsigned long long sub[kSubCap];       // the level-2 boundary bin
    unsigned hist2[kHistBins];             // level-2 histogram (single-CTA selection)
    unsigned part[256];
    unsigned rh[256];                      // radix fallback digit histogram
    unsigned bin, above, count;            // result of block_find_bin / find_bin_warp
    unsigned fbin, fabove, fcount;         // the 16-bit boundary bin, the count above it, its count
    unsigned n_a, n_b, n_s, n_up;
    unsigned last, flags, maxb;
    unsigned long long prefix;
    unsigned done;
    unsigned long long red[64];            // per-warp partial minima / maxima
    unsigned wsum[32];                     // per-warp scan totals
    unsigned wcnt[32];                     // per-warp counts
};

// Per-query words of a multi-CTA selection in global memory (zeroed before the launch).
enum SelCounter { kCntArrive = 0, kCntTicket = 1, kCntSample = 2, kCntWords = 8 };
constexpr int kMaxSelCtas = 256;   // CTAs of one query in a multi-CTA selection (per-CTA list words)
constexpr int kSampleUnion = 1024; // sample keys the CTAs of one query publish (at most)

// Composites per query of each multi-CTA list region: CTA g of a query writes at g * stride, where
// stride is at most its score range per + 1 (per = max(ceil(n_vis / G), 64), G <= ceil(ld / 64) and
// G <= 256): G * (per + 1) is at most ld + 2 G <= ld + 512 when per > 64, and 65 G <= 1.02 ld + 65
// when per = 64, so 2 ld + 512 always suffices.
__host__ __device__ constexpr long long sel_list_cap(long long ld) { return 2 * ld + 512; }

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Ticket of a CTA (one thread, after a bar.sync that orders its CTA's writes): a release-acquire
// atomic increment; true on the CTA that completes the count, which then sees every CTA's writes.
__device__ __forceinline__ bool take_ticket(unsigned *ctr, int n_ctas) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(ctr) : "memory");
    return old == static_cast<unsigned>(n_ctas - 1);
}

// Grid barrier of the n_ctas CTAs of one query (one thread per CTA, after a bar.sync; every CTA
// resident): release-increment, then acquire-poll until all have arrived. Returns false if the
// wait gave up after kSelWaitLimit polls.
__device__ __forceinline__ bool grid_barrier(unsigned *ctr, int n_ctas) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
    const uint32_t limit = *static_cast<volatile uint32_t *>(&g_cross_cta_wait_limit);
    for (uint32_t it = 0; it < limit; it++) {
        if (ld_acquire(ctr) >= static_cast<unsigned>(n_ctas)) return true;
        __nanosleep(32);
    }
    return false;
}

// On warp 0 only: in a histogram of `nbins` bins (a multiple of 32) the highest bin whose suffix
// count (it and all higher bins) reaches k; writes s.bin, s.above (count in higher bins) and
// s.count (the bin's own count). Requires k <= total.
__device__ __forceinline__ void find_bin_warp(const unsigned *hist, int nbins, unsigned k, SelShared &s) {
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
                s.bin = static_cast<unsigned>(per * lane + j);
                s.above = above;
                s.count = c;
                break;
            }
            above += c;
        }
    }
}

// Block-wide boundary search in a 2048-bin shared histogram (blockDim.x >= 256, every thread
// calls): 256 partial sums of 8 bins, then warp 0 finds the partial and the bin inside it.
// Requires 1 <= k <= total; the result is in s.bin / s.above / s.count after the call.
__device__ __forceinline__ void block_find_bin(const unsigned *hist, unsigned k, SelShared &s) {
    const int t = threadIdx.x;
    if (t == 0) { s.bin = 0; s.above = 0; s.count = 0; }
    if (t < 256) {
        const uint4 a = reinterpret_cast<const uint4 *>(hist)[2 * t];
        const uint4 b = reinterpret_cast<const uint4 *>(hist)[2 * t + 1];
        s.part[t] = (a.x + a.y) + (a.z + a.w) + (b.x + b.y) + (b.z + b.w);
    }
    __syncthreads();
    if (t < 32) {
        const int lane = t;
        unsigned pv[8], lane_sum = 0;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            pv[j] = s.part[8 * lane + j];
            lane_sum += pv[j];
        }
        unsigned suf = lane_sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += v;
        }
        unsigned above = suf - lane_sum;
        if (above < k && k <= suf) {
            int p = 0;
#pragma unroll
            for (int j = 7; j >= 0; j--) {
                if (above + pv[j] >= k) { p = 8 * lane + j; break; }
                above += pv[j];
            }
            const uint4 a = reinterpret_cast<const uint4 *>(hist)[2 * p];
            const uint4 b = reinterpret_cast<const uint4 *>(hist)[2 * p + 1];
            const unsigned hv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 7; j >= 0; j--) {
                if (above + hv[j] >= k) {
                    s.bin = static_cast<unsigned>(8 * p + j);
                    s.above = above;
                    s.count = hv[j];
                    break;
                }
                above += hv[j];
            }
        }
    }
    __syncthreads();
}

// Warp-aggregated append of the lanes with `take` to list[*counter ...] (capacity cap); returns
// the lane's slot (>= cap means dropped).
__device__ __forceinline__ unsigned warp_append(bool take, unsigned *counter) {
    const int lane = threadIdx.x & 31;
    const unsigned m = __ballot_sync(0xffffffffu, take);
    unsigned p = 0;
    if (lane == 0 && m) p = atomicAdd(counter, __popc(m));
    p = __shfl_sync(0xffffffffu, p, 0);
    return p + __popc(m & ((1u << lane) - 1));
}

// The same for two lists at once (both atomics in flight together): slots in ra / rb.
__device__ __forceinline__ void warp_append2(bool ta, unsigned *ca, bool tb, unsigned *cb, unsigned &ra,
                                             unsigned &rb) {
    const int lane = threadIdx.x & 31;
    const unsigned ma = __ballot_sync(0xffffffffu, ta), mb = __ballot_sync(0xffffffffu, tb);
    unsigned pa = 0, pb = 0;
    if (lane == 0) {
        if (ma) pa = atomicAdd(ca, __popc(ma));
        if (mb) pb = atomicAdd(cb, __popc(mb));
    }
    pa = __shfl_sync(0xffffffffu, pa, 0);
    pb = __shfl_sync(0xffffffffu, pb, 0);
    const unsigned lt = (1u << lane) - 1;
    ra = pa + __popc(ma & lt);
    rb = pb + __popc(mb & lt);
}

// Classify the scores i in [lo, hi) (score_at(i) -> fp32; every thread of the block calls):
// keys above bin bstar (or every key when bstar < 0) go to s.cand (list A), keys of bin bstar to
// s.bnd (list B) with their level-2 digit counted in hist2 (shared or global memory).
template <typename ScoreAt>
__device__ __forceinline__ void classify_range(const ScoreAt &score_at, int lo, int hi, int bstar,
                                               unsigned *hist2, SelShared &s, int shift = 32 - kHistBitsTop) {
    const int T = blockDim.x;
#pragma unroll 1
    for (int b0 = lo; b0 < hi; b0 += T) {
        const int i = b0 + static_cast<int>(threadIdx.x);
        const bool ok = i < hi;
        const uint32_t key = ok ? score_key(score_at(i)) : 0u;
        const int d = static_cast<int>(key >> shift);
        const bool a = ok && (bstar < 0 || d > bstar);
        const bool b = ok && bstar >= 0 && d == bstar;
        if (!__any_sync(0xffffffffu, a || b)) continue;
        unsigned ra, rb;
        warp_append2(a, &s.n_a, b, &s.n_b, ra, rb);
        const unsigned long long c = compose(key, i);
        if (a && ra < static_cast<unsigned>(kMaxSelect)) s.cand[ra] = c;
        if (b) {
            if (rb < static_cast<unsigned>(kBoundCap)) s.bnd[rb] = c;
            if (hist2) atomicAdd(&hist2[(c >> kShift2) & (kHistBins - 1)], 1u);
        }
    }
}

// Radix selection of the k largest composites among entries sharing `prefix` on the leading
// known_bits bits; get(i) for i < m gives an entry (0 = none). On return s.prefix / s.done
// describe the boundary: the selection is every entry e with (e & ~0 << (64 - done)) >= prefix.
template <typename Get>
__device__ __noinline__ void radix_select(const Get &get, int m, unsigned k, int known_bits,
                                             unsigned long long prefix, SelShared &s) {
    const int tid = threadIdx.x;
    unsigned long long mask = known_bits > 0 ? ~0ull << (64 - known_bits) : 0ull;
    int bits = known_bits;
    while (bits < 64) {
        const int width = min(8, 64 - bits);
        const int shift = 64 - bits - width;
        for (int i = tid; i < 256; i += blockDim.x) s.rh[i] = 0;
        if (tid == 0) { s.bin = 0; s.above = 0; s.count = 0; }
        __syncthreads();
        for (int i = tid; i < m; i += blockDim.x) {
            const unsigned long long c = get(i);
            if (c != 0ull && (c & mask) == prefix)
                atomicAdd(&s.rh[static_cast<uint32_t>((c >> shift) & ((1u << width) - 1))], 1u);
        }
        __syncthreads();
        if (tid < 32) find_bin_warp(s.rh, 256, k, s);
        __syncthreads();
        const unsigned d = s.bin, above = s.above, in_bin = s.count;
        prefix |= static_cast<unsigned long long>(d) << shift;
        mask |= static_cast<unsigned long long>((1u << width) - 1) << shift;
        bits += width;
        k -= above;
        __syncthreads();
        if (k == in_bin) break;  // the whole digit is taken: resolved
    }
    if (tid == 0) { s.prefix = prefix; s.done = static_cast<unsigned>(bits); }
    __syncthreads();
}

// Append every entry with get(i) != 0 and (c & msk) >= pre to s.cand[base ...].
template <typename Get>
__device__ __noinline__ void collect_from(const Get &get, int m, unsigned long long msk,
                                             unsigned long long pre, unsigned base, SelShared &s) {
    if (threadIdx.x == 0) s.n_s = 0;
    __syncthreads();
    for (int b0 = 0; b0 < m; b0 += blockDim.x) {
        const int i = b0 + static_cast<int>(threadIdx.x);
        const unsigned long long c = i < m ? get(i) : 0ull;
        const bool take = c != 0ull && (c & msk) >= pre;
        const unsigned pos = base + warp_append(take, &s.n_s);
        if (take && pos < static_cast<unsigned>(kMaxSelect)) s.cand[pos] = c;
    }
    __syncthreads();
}

// Bitonic sort of a[0 .. count) (count <= 2048, blockDim.x a multiple of 32 with
// blockDim.x * 4 >= 2048), descending, in place. Elements live in registers (up to 4 per
// thread at positions i * blockDim + tid); exchanges at distance < 32 use warp shuffles, larger
// ones go through shared memory.
static __device__ __noinline__ void sort_desc(unsigned long long *a, int count) {
    const int T = blockDim.x, t = threadIdx.x;
    int P2 = 32;
    while (P2 < count) P2 <<= 1;
    unsigned long long e[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int x = i * T + t;
        e[i] = x < count ? a[x] : 0ull;   // 0 sorts last
    }
    for (int k = 2; k <= P2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= 32) {
                __syncthreads();
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int x = i * T + t;
                    if (x < P2) a[x] = e[i];
                }
                __syncthreads();
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int x = i * T + t;
                    if (x < P2) {
                        const unsigned long long o = a[x ^ j];
                        const bool keep_max = ((x & k) == 0) == ((x & j) == 0);
                        e[i] = keep_max ? (e[i] > o ? e[i] : o) : (e[i] < o ? e[i] : o);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int x = i * T + t;
                    if (i * T < P2) {   // whole warps in or out: the shuffle is warp-uniform
                        const unsigned long long o = __shfl_xor_sync(0xffffffffu, e[i], j);
                        const bool keep_max = ((x & k) == 0) == ((x & j) == 0);
                        e[i] = keep_max ? (e[i] > o ? e[i] : o) : (e[i] < o ? e[i] : o);
                    }
                }
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int x = i * T + t;
        if (x < count) a[x] = e[i];
    }
    __syncthreads();
}

// Sort of a[0 .. count) (unique composites, count <= 2048), descending, in place, by buckets:
// each composite gets a bucket linear in its distance from the smallest one (the distance shifted
// right until the largest fits 2048 buckets: monotone, so a higher bucket holds only larger
// composites, and at least 1024 buckets are in use); a suffix scan of the
// bucket counts gives every bucket its output range, the entries are scattered into their bucket
// and ranked inside it by counting. Buckets stay small for any spread of scores; if one holds
// more than kMaxBucket entries (extreme clustering) the bitonic sort runs instead.
// Scratch: s.hist2 (counts), s.bnd (16 KB of scattered entries, then offsets and cursors).
// Requires blockDim.x == 512 (one thread per 4 of the 2048 buckets in the scan).
constexpr int kMaxBucket = 96;
__device__ __forceinline__ void sort_selected(unsigned long long *a, int count, SelShared &s) {
    const int T = blockDim.x, t = threadIdx.x, lane = t & 31, warp = t >> 5, nw = T >> 5;
    if (count <= 1) return;
    unsigned long long *tmp = s.bnd;                                        // [2048]
    unsigned *off = reinterpret_cast<unsigned *>(s.bnd + kMaxSelect);       // [2048]
    unsigned *cur = off + kHistBins;                                        // [2048]
    unsigned long long lo = ~0ull, hi = 0ull;
#pragma unroll 1
    for (int x = t; x < count; x += T) {
        const unsigned long long e = a[x];
        lo = e < lo ? e : lo;
        hi = e > hi ? e : hi;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long l2 = __shfl_xor_sync(0xffffffffu, lo, o), h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
    }
    if (lane == 0) { s.red[warp] = lo; s.red[32 + warp] = hi; }
    if (t == 0) s.maxb = 0;
#pragma unroll 1
    for (int i = t; i < kHistBins; i += T) { s.hist2[i] = 0; cur[i] = 0; }
    __syncthreads();
    lo = lane < nw ? s.red[lane] : ~0ull;   // every warp reduces the per-warp extremes itself
    hi = lane < nw ? s.red[32 + lane] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long l2 = __shfl_xor_sync(0xffffffffu, lo, o), h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
    }
    // bucket = (e - lo) >> sh with the smallest shift that maps hi into the 2048 buckets
    const int sh = max(0, 64 - __clzll(static_cast<long long>(hi - lo)) - kHistBitsTop);
#pragma unroll 1
    for (int x = t; x < count; x += T) atomicAdd(&s.hist2[static_cast<int>((a[x] - lo) >> sh)], 1u);
    __syncthreads();
    // suffix scan: off[b] = number of entries in buckets above b (thread t owns buckets
    // 2047 - 4t .. 2044 - 4t, so that a prefix over threads is a suffix over buckets)
    const uint4 q = reinterpret_cast<const uint4 *>(s.hist2)[(kHistBins / 4 - 1) - t];
    const unsigned tsum = (q.x + q.y) + (q.z + q.w);
    unsigned vmax = max(max(q.x, q.y), max(q.z, q.w));
    unsigned incl = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
        vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 31) s.wsum[warp] = incl;
    if (lane == 0) atomicMax(&s.maxb, vmax);
    __syncthreads();
    unsigned before = lane < warp ? s.wsum[lane] : 0u;   // totals of the warps before this one
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
    const unsigned run = before + incl - tsum;
    const int b0 = kHistBins - 1 - 4 * t;
    off[b0] = run;
    off[b0 - 1] = run + q.w;
    off[b0 - 2] = run + q.w + q.z;
    off[b0 - 3] = run + q.w + q.z + q.y;
    const bool small = s.maxb <= static_cast<unsigned>(kMaxBucket);
    __syncthreads();
    if (!small) {
        sort_desc(a, count);
        return;
    }
#pragma unroll 1
    for (int x = t; x < count; x += T) {   // scatter into the buckets
        const unsigned long long e = a[x];
        const int bk = static_cast<int>((e - lo) >> sh);
        tmp[off[bk] + atomicAdd(&cur[bk], 1u)] = e;
    }
    __syncthreads();
#pragma unroll 1
    for (int p = t; p < count; p += T) {   // rank inside the bucket
        const unsigned long long e = tmp[p];
        const int bk = static_cast<int>((e - lo) >> sh);
        const unsigned start = off[bk], n = s.hist2[bk];
        unsigned rank = start;
#pragma unroll 1
        for (unsigned r = start; r < start + n; r++) rank += tmp[r] > e;
        a[rank] = e;
    }
    __syncthreads();
}

// Finish a selection whose lists are on chip: s.cand[0 .. nA) holds list A, s.bnd[0 .. nB)
// list B when b_complete (else list B is only reachable through get_b over m_b entries: every
// score of the row, with 0 returned for keys outside bin bstar), hist2 its complete level-2
// histogram.
// Leaves the count = min(select_k, n_vis) selected composites sorted in s.cand.
template <typename GetB>
__device__ __forceinline__ void finish_selection(unsigned count, unsigned nA, unsigned nB, bool b_complete,
                                                 int bstar, const unsigned *hist2, const GetB &get_b,
                                                 int m_b, SelShared &s) {
    const int tid = threadIdx.x;
    const unsigned need = count > nA ? count - nA : 0u;
    if (need > 0) {
        const unsigned long long top = static_cast<unsigned long long>(bstar) << (64 - kHistBitsTop);
        if (b_complete && nB == need) {
#pragma unroll 1
            for (unsigned i = tid; i < nB; i += blockDim.x)
                if (nA + i < static_cast<unsigned>(kMaxSelect)) s.cand[nA + i] = s.bnd[i];
            __syncthreads();
        } else if (b_complete) {
            block_find_bin(hist2, need, s);
            const unsigned b2 = s.bin, m2 = s.count;
            const bool small = m2 <= static_cast<unsigned>(kSubCap);
            if (tid == 0) { s.n_up = 0; s.n_s = 0; }
            __syncthreads();
            if (small) {
                // each warp compacts the entries above the sub-bin of its contiguous chunk of list
                // B in place (no shared counter), then moves them behind list A
                const int lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
                const unsigned chunk = (nB + nw - 1) / nw, c0 = min(nB, warp * chunk), c1 = min(nB, c0 + chunk);
                unsigned nup = 0;
#pragma unroll 1
                for (unsigned b0 = c0; b0 < c1; b0 += 32) {
                    const unsigned i = b0 + lane;
                    const unsigned long long x = i < c1 ? s.bnd[i] : 0ull;
                    const unsigned d = static_cast<unsigned>((x >> kShift2) & (kHistBins - 1));
                    const bool up = i < c1 && d > b2;
                    const unsigned m = __ballot_sync(0xffffffffu, up);
                    if (up) s.bnd[c0 + nup + __popc(m & ((1u << lane) - 1))] = x;   // never past i
                    nup += __popc(m);
                    if (i < c1 && d == b2) {   // the sub-bin itself (a handful of entries)
                        const unsigned re = atomicAdd(&s.n_s, 1u);
                        if (re < static_cast<unsigned>(kSubCap)) s.sub[re] = x;
                    }
                }
                if (lane == 0) s.wcnt[warp] = nup;
                __syncthreads();
                unsigned before = lane < nw && lane < warp ? s.wcnt[lane] : 0u;
                unsigned total = lane < nw ? s.wcnt[lane] : 0u;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    before += __shfl_xor_sync(0xffffffffu, before, o);
                    total += __shfl_xor_sync(0xffffffffu, total, o);
                }
#pragma unroll 1
                for (unsigned k = lane; k < nup; k += 32)
                    if (nA + before + k < static_cast<unsigned>(kMaxSelect)) s.cand[nA + before + k] = s.bnd[c0 + k];
                if (tid == 0) s.n_up = total;
                __syncthreads();
                const unsigned got = min(s.n_up, need);
                const unsigned need2 = need - got, base2 = nA + got;
#pragma unroll 1
                for (unsigned i = tid; i < m2; i += blockDim.x) {   // rank inside the sub-bin
                    const unsigned long long x = s.sub[i];
                    unsigned rank = 0;
#pragma unroll 1
                    for (unsigned j = 0; j < m2; j++) rank += s.sub[j] > x;
                    if (rank < need2 && base2 + rank < static_cast<unsigned>(kMaxSelect)) s.cand[base2 + rank] = x;
                }
                __syncthreads();
            } else {   // a large sub-bin (ties at the boundary): radix selection over list B
                auto get = [&](int i) { return s.bnd[i]; };
                radix_select(get, static_cast<int>(nB), need, kHistBitsTop, top, s);
                collect_from(get, static_cast<int>(nB), ~0ull << (64 - s.done), s.prefix, nA, s);
            }
        } else {   // list B did not fit on chip: radix selection straight from its source
            radix_select(get_b, m_b, need, kHistBitsTop, top, s);
            collect_from(get_b, m_b, ~0ull << (64 - s.done), s.prefix, nA, s);
        }
    }
    sort_selected(s.cand, static_cast<int>(count), s);
}

// Multi-CTA selection, after every CTA of the query has classified its slice into s.cand /
// s.bnd (level-2 digits counted straight into the global hist2): CTA g writes its lists to its
// own regions (al / bl + g * stride) and its list sizes to words[g] -- no shared counters --,
// takes a ticket, and the last CTA to finish gathers every CTA's lists and hist2 back on chip.
// Returns true on that CTA (with nA, nB, b_complete set), false elsewhere. Every thread calls it;
// requires n_ctas <= kMaxSelCtas.
constexpr int kGatherK = 10;   // list slots (CTA, entry < 32) per thread gathered in one round trip
__device__ __forceinline__ bool merge_lists_multi(unsigned *cnt, unsigned *words, unsigned long long *al,
                                                  unsigned long long *bl, int stride, const unsigned *ghist2,
                                                  int n_ctas, unsigned &nA, unsigned &nB, bool &b_complete,
                                                  SelShared &s) {
    const int tid = threadIdx.x, g = blockIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const unsigned la = min(s.n_a, static_cast<unsigned>(kMaxSelect));
    const unsigned lb = min(s.n_b, static_cast<unsigned>(kBoundCap));
    unsigned long long *my_a = al + static_cast<long long>(g) * stride;
    unsigned long long *my_b = bl + static_cast<long long>(g) * stride;
#pragma unroll 1
    for (unsigned i = tid; i < la; i += blockDim.x) my_a[i] = s.cand[i];
#pragma unroll 1
    for (unsigned i = tid; i < lb; i += blockDim.x) my_b[i] = s.bnd[i];
    if (tid == 0) words[g] = la | (lb << 11) | (s.n_b > static_cast<unsigned>(kBoundCap) ? 1u << 24 : 0u);
    __syncthreads();
    if (tid == 0)   // release this CTA's lists and take the ticket; the last CTA acquires everyone's
        s.last = take_ticket(&cnt[kCntTicket], n_ctas);
    __syncthreads();
    if (!s.last) return false;
    if (warp == 0) {
        // every CTA's list sizes -> exclusive offsets of both lists (one packed 64-bit scan), the
        // totals, the overflow flag and the longest list
        constexpr int kPer = kMaxSelCtas / 32;
        unsigned long long v[kPer], sum = 0ull;
        unsigned flags = 0, mx = 0;
#pragma unroll
        for (int j = 0; j < kPer; j++) {
            const int c = lane * kPer + j;
            const unsigned w = c < n_ctas ? __ldcg(&words[c]) : 0u;
            const unsigned a = w & 2047u, b = (w >> 11) & 8191u;
            flags |= w >> 24;
            mx = max(mx, max(a, b));
            v[j] = a | (static_cast<unsigned long long>(b) << 32);
            sum += v[j];
        }
        unsigned long long incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
            flags |= __shfl_xor_sync(0xffffffffu, flags, o);
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        unsigned long long run = incl - sum;
#pragma unroll
        for (int j = 0; j < kPer; j++) {
            const int c = lane * kPer + j;
            if (c < n_ctas) {
                s.part[c] = static_cast<unsigned>(run);
                s.rh[c] = static_cast<unsigned>(run >> 32);
            }
            run += v[j];
        }
        if (lane == 31) {
            s.wsum[0] = static_cast<unsigned>(incl);
            s.wsum[1] = static_cast<unsigned>(incl >> 32);
            s.flags = flags;
            s.maxb = mx;
        }
    } else if (ghist2) {   // meanwhile the other warps fetch the level-2 histogram
#pragma unroll 1
        for (int i = tid - 32; i < kHistBins / 4; i += blockDim.x - 32)
            reinterpret_cast<uint4 *>(s.hist2)[i] = __ldcg(reinterpret_cast<const uint4 *>(ghist2) + i);
    }
    __syncthreads();
    nA = min(s.wsum[0], static_cast<unsigned>(kMaxSelect));
    nB = s.wsum[1];
    b_complete = s.flags == 0u && nB <= static_cast<unsigned>(kBoundCap);
    const unsigned totB = b_complete ? nB : 0u;
    auto range = [&](const unsigned *offs, unsigned total, int c, unsigned &o, unsigned &n) {
        o = offs[c];
        n = (c + 1 < n_ctas ? offs[c + 1] : total) - o;
    };
    {   // slot q = (CTA q / 32, entry q % 32): all loads of a thread first, then the stores
        unsigned long long va[kGatherK], vb[kGatherK];
        unsigned da[kGatherK], db[kGatherK];
#pragma unroll
        for (int k = 0; k < kGatherK; k++) {
            const int q = tid + k * blockDim.x, c = q >> 5;
            const unsigned j = q & 31;
            va[k] = 0ull;
            vb[k] = 0ull;
            da[k] = ~0u;
            db[k] = ~0u;
            if (c < n_ctas) {
                unsigned oa, na, ob, nb;
                range(s.part, nA, c, oa, na);
                range(s.rh, totB, c, ob, nb);
                if (j < na) { va[k] = __ldcg(al + static_cast<long long>(c) * stride + j); da[k] = oa + j; }
                if (b_complete && j < nb) { vb[k] = __ldcg(bl + static_cast<long long>(c) * stride + j); db[k] = ob + j; }
            }
        }
#pragma unroll
        for (int k = 0; k < kGatherK; k++) {
            if (da[k] < static_cast<unsigned>(kMaxSelect)) s.cand[da[k]] = va[k];
            if (db[k] != ~0u) s.bnd[db[k]] = vb[k];
        }
    }
    const int done_ctas = kGatherK * static_cast<int>(blockDim.x) / 32;
    if (s.maxb > 32u || n_ctas > done_ctas) {   // entries past the 32nd of a CTA, CTAs past the slots
#pragma unroll 1
        for (int c = warp; c < n_ctas; c += nw) {
            unsigned oa, na, ob = 0, nb = 0;
            range(s.part, nA, c, oa, na);
            if (b_complete) range(s.rh, totB, c, ob, nb);
#pragma unroll 1
            for (unsigned j = (c < done_ctas ? 32u : 0u) + lane; j < max(na, nb); j += 32) {
                if (j < na && oa + j < static_cast<unsigned>(kMaxSelect))
                    s.cand[oa + j] = __ldcg(al + static_cast<long long>(c) * stride + j);
                if (j < nb) s.bnd[ob + j] = __ldcg(bl + static_cast<long long>(c) * stride + j);
            }
        }
    }
    __syncthreads();
    return true;
}

// Writes the selection's pool ids (s.cand[0 .. count), sorted) and -1 up to select_k.
__device__ __forceinline__ void write_selection(int32_t *row, int select_k, unsigned count, const SelShared &s) {
    for (int x = threadIdx.x; x < select_k; x += blockDim.x)
        row[x] = static_cast<unsigned>(x) < count ? id_of(s.cand[x]) : GLM_INVALID;
}

}  // namespace glm
