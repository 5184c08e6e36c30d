// index_select_tc.cu -- relu head-weighted index scores on the sm_100a tensor cores, fused with
// the top-k pool selection and its expansion into token indices and cache rows
// ("Module glm5next_dsa_ref": index_scores -- matmul -> relu -> head-weighted sum --, topk_pools
// and expand_selection; "GLM-5.3-Flash" pypto-lib page, 'Checkpoint shape': indexer 32 heads x 128):
//     score[n][p] = sum_h w[n][h] * max(0, sum_d q_idx[n][h][d] * pooled[b][p][d])
//
// Grid (G, n_q): CTA g of query n owns a contiguous range of the query's visible pools.
// Phase 1, scoring -- a warp-specialised pipeline over chunks of 64 pools, every hand-off an mbarrier:
//   * producer (warp 0): one 1-D bulk copy per chunk (64 pool rows, 32 KB, contiguous) into a ring
//     of 4 slots (128 KB per SM in flight: a fifth slot streamed no faster and made the CTAs'
//     later round trips, which queue behind the bulk data bound for the same SM, slower);
//   * converters (warps 8-15, 8 pool rows of a chunk each): every warp first reads its rows into
//     registers (lane l: dims 4 l .. 4 l + 3 of a row), the warps meet on an mbarrier, and each
//     then rewrites its rows in place as two fp16 terms in the 128-byte swizzle layout: the row
//     scaled by the power of two 2^e_p that puts its largest magnitude in [2^14, 2^15), hi =
//     rn_fp16(x 2^e_p), lo = rn_fp16(x 2^e_p - hi) -- together x to 2^-23 relative --, and 2^-e_p
//     kept for the epilogue. The two terms of each 64-dim K atom sit one above the other (hi rows
//     0-63, lo rows 64-127), so that one MMA of M = 128 covers both. Shared memory sees one copy
//     write, one read and one write of a pool row before the MMA reads: ~2.2 KB per pool;
//   * MMA issuer (warp 1): 8 UMMAs per chunk (M = 128 = the chunk's hi and lo rows, N = 32 heads,
//     K = 16, fp16 operands) into one of two fp32 tensor-memory accumulators -- each tcgen05.mma
//     costs about the same whatever its size here, so the count is what matters; the query block
//     is fp16 with each head scaled by its own power of two (exact for the bf16 query), folded back
//     into the head weight;
//   * epilogue (warps 4-7, one TMEM lane quadrant each): warps 6-7 hold the lo halves of the dots
//     and hand them over through shared memory; warps 4-5 add them to the hi halves, then relu and
//     head weights, the pool's 2^-e_p (both exact powers of two), the score (to global memory and,
//     when the range is short enough, to shared memory), and (one CTA per query) its top-11-bit key
//     digit counted in the CTA's histogram.
// Selection with G = 1: the one CTA selects on chip (histogram boundary bin, lists, sort).
// Selection with G > 1 -- a sample threshold, so that the query's CTAs meet while the keys still
// stream: the first tiles of every CTA's range (about an eighth of it) are a sample of the
// query's scores. While phase 1 runs, warp 2 of each CTA publishes its largest sample keys, the
// CTAs meet (all are resident, at most one per SM; every wait is bounded), and each finds the
// k_s-th largest published key (k_s = 1.5 select_k sample size / visible pools + 16), rounded down
// to 16 bits: the threshold. Scores whose key reaches it are candidates (about 1.5 select_k of
// them): when phase 1 ends, each CTA appends its candidates to the query's list (an offset from a
// counter), the CTAs meet again, and every CTA loads the whole list, ranks its share of it exactly
// (the number of larger composites) and writes the outputs of the select_k best; one CTA writes
// the rest (padding, n_sel, the visible tail). The threshold only prunes: if fewer than select_k
// scores (or more than the list holds on chip) pass it, one CTA selects exactly over every score
// of the row.
// Phase 1 is HBM-bound: 512 bytes of pooled key per pool; the tensor cores run at a few percent.
// With the INT8 indexer state ("GLM-5.3-Flash" pypto-lib page, 'What is quantized': the indexer
// cache in INT8 with one FP32 scale per row) a pool is 128 code bytes plus its scale: a chunk is an
// 8 KB copy, the codes are widened to one exact fp16 term beside them in the slot, and the score is
// multiplied by the pool's scale.
#include "common.cuh"
#include "tc.cuh"
#include "kernels.cuh"
#include "select.cuh"
#include "topk.cuh"

#include <cuda_fp16.h>

namespace glm {

GLM_TL_TABLE(glm_tl_index)

constexpr int kIxThreads = 512;                        // 16 warps, see the roles above
constexpr int kIxTile = 64;                            // pools per chunk (UMMA M)
constexpr int kIxSlots = 4;                            // staging slots, converted in place
constexpr int kIxSlotBytes = kIxTile * kIdxDim * 4;    // 32 KB: 64 fp32 pool rows
constexpr int kIxConv = 8;                             // converter warps (8 rows of a chunk each)
constexpr int kIxAtomBytes = kIxTile * 128;            // 8 KB: one 64-dim K atom of an fp16 term
constexpr int kIxTermBytes = 2 * kIxAtomBytes;         // 16 KB: one fp16 term of a chunk
static_assert(kIxSlots <= 5, "the barrier table holds five slots");
constexpr int kIxPsDepth = kIxSlots + 2;               // ring of the pools' score factors (see converters)
constexpr uint32_t kIxWaitLimit = 1u << 22;

constexpr int kIxLocalCap = 2048;                      // scores of a CTA kept in shared memory
constexpr int kIxSampleTiles = 8;                      // most chunks of a CTA's range in the sample
constexpr int kIxSampleMax = kIxSampleTiles * kIxTile;

struct IxLayout {                                      // offsets from a 1024-byte aligned base
    static constexpr int kSlots = 0;                                  // [kIxSlots][32 KB]
    static constexpr int kQ = kSlots + kIxSlots * kIxSlotBytes;       // 32 heads x 128 dims fp16
    static constexpr int kHist = kQ + kIdxHeads * kIdxDim * 2;        // 2048 uint32
    static constexpr int kLocal = kHist + kHistBins * 4;              // kIxLocalCap fp32 scores
    static constexpr int kW = kLocal + kIxLocalCap * 4;               // 32 fp32 head weights (scaled)
    static constexpr int kPs = kW + kIdxHeads * 4;                    // [kIxPsDepth][64] fp32 score factors
    static constexpr int kXch = kPs + kIxPsDepth * kIxTile * 4;       // [2][64 pools][32 heads] fp32 lo dots
    static constexpr int kBar = kXch + 2 * kIxTile * kIdxHeads * 4;   // 27 mbarriers
    static constexpr int kTmem = kBar + 27 * 8;
    static constexpr int kFlag = kTmem + 16;                          // 8 words, see kFl*
    static constexpr int kSamp = (kFlag + 32 + 15) / 16 * 16;         // the CTA's sample keys
    static constexpr int kScr = kSamp + kIxSampleMax * 4;             // the published keys, staged
    static constexpr int kBytes = kScr + 16 * 4;
    static constexpr int kAlloc = kBytes + 1024;                      // room to align the base
};
static_assert(IxLayout::kScr % 16 == 0, "the threshold's staged keys are read as 16-byte vectors");
static_assert(IxLayout::kAlloc <= 232448, "shared memory of one CTA");
// The selection's working set overlays the staging slots once scoring is over.
static_assert(sizeof(SelShared) <= IxLayout::kQ, "selection working set must fit the staging slots");

// words at IxLayout::kFlag
constexpr int kFlThr = 0;       // the sample threshold: a candidate's key is at least this
constexpr int kFlWait = 1;      // a wait on the query's other CTAs gave up

// mbarrier indices
constexpr int kBarStFull = 0;     // [kIxSlots <= 5] slot filled (producer, tx bytes)
constexpr int kBarStRead = 5;     // [kIxSlots] slot read into registers (8 converter warps)
constexpr int kBarStConv = 10;    // [kIxSlots] slot converted in place (8 converter warps)
constexpr int kBarStEmpty = 15;   // [kIxSlots] slot read by the MMAs (commit)
constexpr int kBarAccFull = 20;   // [2] accumulator ready (commit)
constexpr int kBarAccEmpty = 22;  // [2] accumulator read (4 epilogue warps)
constexpr int kBarSample = 24;    // the sample keys are in shared memory (2 epilogue warps)
constexpr int kBarXch = 25;       // [2] the lo dots of an accumulator are in the exchange buffer (2 warps)

__device__ __forceinline__ uint32_t f16x2_rn(float a, float b) {   // .x = a (low half)
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}
__device__ __forceinline__ float f16_lo_f(uint32_t p) { return __half2float(__ushort_as_half(static_cast<unsigned short>(p & 0xffffu))); }
__device__ __forceinline__ float f16_hi_f(uint32_t p) { return __half2float(__ushort_as_half(static_cast<unsigned short>(p >> 16))); }
// Four int8 codes as four exact fp16 values (1024 + code + 128 built as fp16 bits, minus 1152).
__device__ __forceinline__ uint2 codes_to_f16x4(uint32_t w) {
    const uint32_t t = w ^ 0x80808080u;
    const uint32_t a = __byte_perm(t, 0x64646464u, 0x5140u), b = __byte_perm(t, 0x64646464u, 0x5342u);
    uint2 r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r.x) : "r"(a), "r"(0x64806480u));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r.y) : "r"(b), "r"(0x64806480u));
    return r;
}
// The exponent e that puts a nonzero magnitude m in [2^14, 2^15) once scaled by 2^e (clamped so
// that 2^e and 2^-e are normal floats); 0 for m = 0.
__device__ __forceinline__ int pow2_exponent(float m) {
    if (!(m > 0.0f)) return 0;
    const int E = static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127;
    return min(120, max(-120, 14 - E));
}
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// The k-th largest sample key of a query (warp 2 of each of its n_ctas CTAs): CTA g publishes
// the r largest of its n_samp sample keys (r a multiple of 4; 0 where it has fewer) at gs + g r --
// lane 0 stores them, then releases them as it arrives at the meeting word *ctr --, the CTAs meet,
// and each reads the n_ctas r published keys (at most kSampleUnion, eight 16-byte loads per lane)
// and finds the k-th largest, rounded down to its top kThrBits bits, by a binary search on the
// key bits (stage: kPubMax words of shared memory). The published keys are a subset of the
// sample, so the result is at most the sample's k-th largest key: a threshold that lets through
// at least as many scores. Returns 0 -- every score passes -- when fewer than k keys are
// published. ok turns false on lane 0 if the wait gave up.
constexpr int kPubMax = 16;   // published keys per CTA, at most
constexpr int kThrBits = 16;  // bits of the threshold key that are searched (the rest are 0)
__device__ __noinline__ unsigned sample_threshold(const unsigned *samp, int n_samp, int r, unsigned k,
                                                  unsigned *gs, int g, unsigned *ctr, int n_ctas,
                                                  unsigned *stage, bool &ok) {
    const int lane = threadIdx.x & 31;
    // this CTA's r largest keys: r rounds of a warp-wide maximum over the lanes' own keys
    unsigned kv[kIxSampleMax / 32];
#pragma unroll
    for (int j = 0; j < kIxSampleMax / 32; j++) {
        const int i = j * 32 + lane;
        kv[j] = i < n_samp ? samp[i] : 0u;
    }
    unsigned *top = stage;   // the r keys, largest first
#pragma unroll 1
    for (int q = 0; q < r; q++) {
        unsigned m = 0u;
#pragma unroll
        for (int j = 0; j < kIxSampleMax / 32; j++) m = max(m, kv[j]);
        const unsigned M = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) top[q] = M;
        const unsigned own = __ballot_sync(0xffffffffu, m == M);
        if (lane == __ffs(own) - 1) {   // that lane drops one copy of M
            bool done = false;
#pragma unroll
            for (int j = 0; j < kIxSampleMax / 32; j++)
                if (!done && kv[j] == M) { kv[j] = 0u; done = true; }
        }
    }
    if (lane == 0) {
#pragma unroll 1
        for (int q = 0; q < r; q += 4)
            *reinterpret_cast<uint4 *>(gs + static_cast<int64_t>(g) * r + q) = *reinterpret_cast<const uint4 *>(top + q);
        if (!grid_barrier(ctr, n_ctas)) ok = false;
        GLM_TL_AT(glm_tl_index, 14, 64);
    }
    __syncwarp();   // the other lanes wait for lane 0's acquire
    const int U = n_ctas * r;
    if (static_cast<unsigned>(U) < k) return 0u;
    uint4 u[kSampleUnion / 128];
#pragma unroll
    for (int j = 0; j < kSampleUnion / 128; j++) {
        const int i = j * 32 + lane;   // 16-byte piece: keys 4 i .. 4 i + 3
        u[j] = 4 * i < U ? __ldcg(reinterpret_cast<const uint4 *>(gs) + i) : make_uint4(0u, 0u, 0u, 0u);
    }
    // the k-th largest published key, to 16 bits (rounded down: a threshold at most that key), by
    // a binary search on its bits: keep each bit if at least k keys reach the prefix with it set
    unsigned prefix = 0u;
#pragma unroll 1
    for (int bit = 31; bit >= 32 - kThrBits; bit--) {
        const unsigned cand = prefix | (1u << bit);
        unsigned c = 0u;
#pragma unroll
        for (int j = 0; j < kSampleUnion / 128; j++)   // (absent keys are 0 and never count)
            c += (u[j].x >= cand) + (u[j].y >= cand) + (u[j].z >= cand) + (u[j].w >= cand);
        if (__reduce_add_sync(0xffffffffu, c) >= k) prefix = cand;
    }
    return prefix;
}

// The cache row of padded token t of sequence b (the slot map's entry; the token itself without a
// slot map), -1 where there is none.
__device__ __forceinline__ int32_t row_of(const IxSelectArgs &sel, int b, long long t) {
    long long rv = t;
    if (sel.slot_map) rv = (t >= 0 && t < sel.ld_slot) ? sel.slot_map[static_cast<int64_t>(b) * sel.ld_slot + t] : -1ll;
    return (rv >= 0 && rv <= 0x7fffffffll) ? static_cast<int32_t>(rv) : GLM_INVALID;
}

// The outputs of the selected pool p of rank r (r < the selection's count): its top-k entry and
// its kKpool expanded token / cache-row entries (the rules of expand_selection). Lanes 0 ..
// kKpool of a warp write them.
__device__ __forceinline__ void write_ranked(const IxSelectArgs &sel, int n, int b, int pb, unsigned r, int p,
                                             int lane) {
    if (lane == kKpool) sel.topk[static_cast<int64_t>(n) * sel.select_k + r] = p;
    if (lane < kKpool) {
        const int64_t j = static_cast<int64_t>(n) * sel.out_width + kKpool * static_cast<int64_t>(r) + lane;
        const int t = pb + kKpool * p + lane;
        if (sel.tok) sel.tok[j] = t;
        if (sel.rows) sel.rows[j] = row_of(sel, b, t);
    }
}

// The outputs no selected pool owns (one CTA of a query, count >= 1 pools selected): the top-k
// row's -1 padding, n_sel, and the expanded entries past the selected pools -- the visible tail,
// then -1 up to out_width.
__device__ __forceinline__ void write_unranked(const IxSelectArgs &sel, int n, int b, int pb, int seq_len,
                                               int qp, unsigned count) {
    for (int x = static_cast<int>(count) + static_cast<int>(threadIdx.x); x < sel.select_k; x += blockDim.x)
        sel.topk[static_cast<int64_t>(n) * sel.select_k + x] = GLM_INVALID;
    if (threadIdx.x == 0 && sel.n_sel) sel.n_sel[n] = static_cast<int32_t>(count);
    if (!sel.tok && !sel.rows) return;
    const int nvx = visible_pools(pb, seq_len, qp, 0x7fffffffll);   // uncapped, as the expansion defines it
    const int ns = min(static_cast<int>(count), nvx);
    const int last = min(qp, pb + seq_len - 1);                     // the tail stops at the query or the end
    const int tail = max(0, last - (pb + kKpool * nvx) + 1);
    const int n_valid = kKpool * ns + tail;
    for (int j = kKpool * ns + static_cast<int>(threadIdx.x); j < sel.out_width; j += blockDim.x) {
        const int t = j < n_valid ? pb + kKpool * nvx + (j - kKpool * ns) : GLM_INVALID;
        const int64_t o = static_cast<int64_t>(n) * sel.out_width + j;
        if (sel.tok) sel.tok[o] = t;
        if (sel.rows) sel.rows[o] = t >= 0 ? row_of(sel, b, t) : GLM_INVALID;
    }
}

// Write the outputs of a query whose selection is final (s.cand[0 .. count) sorted): the top-k
// row, n_sel, and the expansion into tokens / cache rows (the rules of expand_selection).
__device__ __forceinline__ void write_outputs(const IxSelectArgs &sel, int n, int b, bool valid_b, int pb,
                                              int seq_len, int qp, unsigned count, const SelShared &s) {
    write_selection(sel.topk + static_cast<int64_t>(n) * sel.select_k, sel.select_k, count, s);
    if (threadIdx.x == 0 && sel.n_sel) sel.n_sel[n] = static_cast<int32_t>(count);
    if (!sel.tok && !sel.rows) return;
    const int64_t base = static_cast<int64_t>(n) * sel.out_width;
    int nvx = 0, n_valid = 0, ns = 0;
    if (valid_b) {
        nvx = visible_pools(pb, seq_len, qp, 0x7fffffffll);   // uncapped, as the expansion defines it
        ns = min(static_cast<int>(count), nvx);
        const int last = min(qp, pb + seq_len - 1);            // the tail stops at the query or the end
        const int tail = max(0, last - (pb + kKpool * nvx) + 1);
        n_valid = kKpool * ns + tail;
    }
    constexpr int kU = 5;   // entries per thread in flight (slot-map loads issued together)
    for (int j0 = 0; j0 < sel.out_width; j0 += kU * static_cast<int>(blockDim.x)) {
        int tv[kU];
        long long rv[kU];
#pragma unroll
        for (int u = 0; u < kU; u++) {
            const int j = j0 + u * static_cast<int>(blockDim.x) + static_cast<int>(threadIdx.x);
            int t = GLM_INVALID;
            if (j < kKpool * ns) t = pb + kKpool * id_of(s.cand[j / kKpool]) + (j % kKpool);
            else if (j < n_valid) t = pb + kKpool * nvx + (j - kKpool * ns);
            tv[u] = t;
            rv[u] = t;
            if (sel.rows && sel.slot_map)
                rv[u] = (t >= 0 && t < sel.ld_slot) ? sel.slot_map[static_cast<int64_t>(b) * sel.ld_slot + t] : -1ll;
        }
#pragma unroll
        for (int u = 0; u < kU; u++) {
            const int j = j0 + u * static_cast<int>(blockDim.x) + static_cast<int>(threadIdx.x);
            if (j >= sel.out_width) continue;
            if (sel.tok) sel.tok[base + j] = tv[u];
            if (sel.rows)
                sel.rows[base + j] = (rv[u] >= 0 && rv[u] <= 0x7fffffffll) ? static_cast<int>(rv[u]) : GLM_INVALID;
        }
    }
}

// At most 96 registers (83 used, no spill): a CTA then fits on an SM beside a CTA of the step's
// first kernel, so that the grid can start while that kernel runs. Launched with kIxThreads threads.
// kQ8: the pooled keys are the INT8 indexer state (int8 codes [B][ld][128], one fp32 scale per
// pool): one exact bf16 term per key instead of three, and the score is scaled by the pool's scale.
template <bool kQ8>
__global__ void __maxnreg__(96) index_select_tc_kernel(
    const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
    const void *__restrict__ keys, const float *__restrict__ key_scales, int64_t ld_pools,
    const int32_t *__restrict__ q_seq,
    const int32_t *__restrict__ q_pos, const int32_t *__restrict__ pad,
    const int32_t *__restrict__ len, int batch, float *__restrict__ scores, int fill_invisible,
    IxSelectArgs sel, int *__restrict__ status) {
    constexpr int kElem = kQ8 ? 1 : 4;                            // bytes per key element
    // The next kernel of the stream may launch only once this one's CTAs reach the selection (its
    // CTAs then take the SMs the finished CTAs free). Early mode: wait for the preceding kernel
    // only where its outputs are needed; otherwise at once.
    if (!sel.early) asm volatile("griddepcontrol.wait;" ::: "memory");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *slots = smem + IxLayout::kSlots;
    unsigned char *Qs = smem + IxLayout::kQ;
    float *ps_ring = reinterpret_cast<float *>(smem + IxLayout::kPs);
    unsigned *hist = reinterpret_cast<unsigned *>(smem + IxLayout::kHist);
    float *sloc = reinterpret_cast<float *>(smem + IxLayout::kLocal);
    float *ws = reinterpret_cast<float *>(smem + IxLayout::kW);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + IxLayout::kTmem);
    unsigned *flag = reinterpret_cast<unsigned *>(smem + IxLayout::kFlag);
    unsigned *samp = reinterpret_cast<unsigned *>(smem + IxLayout::kSamp);
    unsigned *scr = reinterpret_cast<unsigned *>(smem + IxLayout::kScr);

    const int n = blockIdx.y, g = blockIdx.x, G = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = q_seq[n];
    const bool valid_b = b >= 0 && b < batch;
    const int pb = valid_b ? pad[b] : 0, seq_len = valid_b ? len[b] : 0, qp = q_pos[n];
    const int n_vis = valid_b ? visible_pools(pb, seq_len, qp, ld_pools) : 0;
    // pools the preceding kernel may still be writing (early mode): [first_new, first_new + new_pools)
    const int first_new = (sel.early && valid_b) ? (sel.new_pool_begin ? max(0, sel.new_pool_begin[b]) : 0) : 0;
    float *srow = scores + static_cast<int64_t>(n) * ld_pools;
    const bool select = sel.topk != nullptr;
    const bool multi = select && G > 1;
    SelShared &s = *reinterpret_cast<SelShared *>(slots);
    GLM_TL(glm_tl_index, 0);
    GLM_TL_SMID(glm_tl_index);

    if (fill_invisible) {  // entries past the visible pools are -inf (split over the CTAs)
        const int64_t rest = ld_pools - n_vis;
        const int64_t share = (rest + G - 1) / G;
        const int64_t f0 = n_vis + static_cast<int64_t>(g) * share;
        const int64_t f1 = min(f0 + share, ld_pools);
        for (int64_t i = f0 + tid; i < f1; i += kIxThreads) srow[i] = -INFINITY;
    }
    if (n_vis == 0) {   // nothing to score or select: CTA 0 writes the empty outputs
        if (sel.early) asm volatile("griddepcontrol.wait;" ::: "memory");
        if (select && g == 0) write_outputs(sel, n, b, valid_b, pb, seq_len, qp, 0u, s);
        return;
    }
    int per = (n_vis + G - 1) / G;
    if (per < kIxTile) per = kIxTile;
    const int lo = min(n_vis, g * per);
    const int hi = min(n_vis, lo + per);
    const bool keep_local = select && per <= kIxLocalCap;
    const int g_eff = (n_vis + per - 1) / per;   // CTAs with a score range
    // multi-CTA sample: the first n_st0 tiles of every CTA's range; m_all keys in all, and the
    // threshold is the k_s-th largest of them (no threshold when the sample is that small)
    const int n_st0 = min(kIxSampleTiles, max(1, (per + 8 * kIxTile - 1) / (8 * kIxTile)));
    const int s0 = n_st0 * kIxTile;
    const long long m_all = static_cast<long long>(g_eff - 1) * min(s0, per) + min(s0, n_vis - (g_eff - 1) * per);
    const long long k_s = (3ll * sel.select_k * m_all + 2ll * n_vis - 1) / (2ll * n_vis) + 16;
    const bool sample = multi && n_vis > sel.select_k && k_s < m_all;
    // keys each CTA publishes for the threshold: enough that their union holds about 2 k_s, a
    // multiple of 4, and at most kSampleUnion in all
    const int r_pub = min(min(kPubMax, (kSampleUnion / max(g_eff, 1)) & ~3),
                          max(4, static_cast<int>((2 * k_s + g_eff - 1) / max(g_eff, 1) + 3) & ~3));
    if (lo < hi) {
    const int n_chunks = (hi - lo + kIxTile - 1) / kIxTile;
    const unsigned char *src = static_cast<const unsigned char *>(keys) +
                               (static_cast<int64_t>(b) * ld_pools + lo) * kIdxDim * kElem;

    const uint32_t bar0 = tc::smem_addr(smem + IxLayout::kBar);
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    const uint32_t slots_addr = tc::smem_addr(slots);
    bool waited_new = !sel.early;   // (producer) the preceding kernel's pools are safe to read
    // the producer's copy of chunk c (waits first for the preceding kernel when the chunk holds a
    // pool it writes)
    auto issue = [&](int c) {
        const int slot = c % kIxSlots;
        const int c0 = lo + c * kIxTile;
        if (!waited_new && c0 + kIxTile > first_new && c0 < first_new + sel.new_pools) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            asm volatile("fence.proxy.async.global;" ::: "memory");
            waited_new = true;
        }
        const uint32_t bytes = static_cast<uint32_t>(min(kIxTile, hi - c0)) * kIdxDim * kElem;
        tc::mbar_arrive_expect_tx(bar(kBarStFull + slot), bytes);
        tc::bulk_g2s(slots_addr + slot * kIxSlotBytes, src + static_cast<int64_t>(c) * kIxTile * kIdxDim * kElem,
                     bytes, bar(kBarStFull + slot));
    };
    // the query block's and head weights' loads go out before the first key copies, which would
    // otherwise queue them behind the whole burst of the query's CTAs
    const uint16_t *qn = q_idx + static_cast<int64_t>(n) * kIdxHeads * kIdxDim;
    const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(qn) + tid);
    const float wv = (tid & 15) == 0 ? __ldg(w + static_cast<int64_t>(n) * kIdxHeads + (tid >> 4)) : 0.0f;
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), 64);
        tc::tmem_relinquish();
        tc::fence_before_sync();
        if (lane == 0) {   // the barriers, then the first copies: the stream starts before the set-up ends
            for (int i = 0; i < kIxSlots; i++) {
                tc::mbar_init(bar(kBarStFull + i), 1);
                tc::mbar_init(bar(kBarStRead + i), kIxConv);
                tc::mbar_init(bar(kBarStConv + i), kIxConv);
                tc::mbar_init(bar(kBarStEmpty + i), 1);
            }
            for (int i = 0; i < 2; i++) tc::mbar_init(bar(kBarAccFull + i), 1);
            for (int i = 0; i < 2; i++) tc::mbar_init(bar(kBarAccEmpty + i), 4);
            for (int i = 0; i < 2; i++) tc::mbar_init(bar(kBarXch + i), 2);
            tc::mbar_init(bar(kBarSample), kQ8 ? 4 : 2);
            tc::mbar_fence_init();
        }
    }
    __syncthreads();   // (the loads above are issued by every thread; the barriers are initialised)
    if (warp == 0 && lane == 0)
        for (int c = 0; c < min(kIxSlots, n_chunks); c++) issue(c);
    // query block as fp16 (core matrices: head group stride 2048 B, dim group 128 B), each head
    // scaled by the power of two 2^f_h that puts its largest magnitude in [2^14, 2^15) -- exact
    // for bf16 values -- and its head weight by 2^-f_h, so that w_h relu(q_h . x) is unchanged:
    // thread t holds dims 8 (t % 16) .. + 7 of head t / 16 (a head's 16 threads share a half-warp)
    {
        const int h = tid >> 4, dg = tid & 15;
        const uint32_t w4[4] = {qv.x, qv.y, qv.z, qv.w};
        unsigned mb = 0u;   // largest |q| bits (bf16 magnitudes order as integers)
#pragma unroll
        for (int e = 0; e < 4; e++) mb = max(mb, max(w4[e] & 0x7fffu, (w4[e] >> 16) & 0x7fffu));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
        const int f = pow2_exponent(__uint_as_float(mb << 16));
        const float sc = pow2f(f);
        uint32_t o4[4];
#pragma unroll
        for (int e = 0; e < 4; e++) o4[e] = f16x2_rn(__uint_as_float(w4[e] << 16) * sc, __uint_as_float(w4[e] & 0xffff0000u) * sc);
        *reinterpret_cast<uint4 *>(Qs + (h >> 3) * 2048 + dg * 128 + (h & 7) * 16) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        if (dg == 0) ws[h] = wv * pow2f(-f);
    }
    if (select && !multi)
        for (int i = tid; i < kHistBins; i += kIxThreads) hist[i] = 0;
    if (tid == 64) {
        flag[kFlThr] = 0;
        flag[kFlWait] = 0;
    }
    tc::fence_proxy_async();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    GLM_TL(glm_tl_index, 1);

    if (warp == 0) {
        // ---------------- producer (the first kIxSlots copies were issued during the set-up) ----------------
        if (lane == 0) {
            for (int c = kIxSlots; c < n_chunks; c++) {
                const int slot = c % kIxSlots;
                if (!tc::mbar_wait(bar(kBarStEmpty + slot), ((c / kIxSlots) - 1) & 1, kIxWaitLimit)) ok = false;
                issue(c);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            // fp32 keys: M = 128, the chunk's hi rows over its lo rows (one K atom = 16 KB); int8 keys:
            // M = 64, the one term at the slot's upper half (one K atom = 8 KB)
            const uint32_t idesc = tc::idesc_f16(kQ8 ? kIxTile : 2 * kIxTile, kIdxHeads, false, false);
            const uint32_t q_addr = tc::smem_addr(Qs);
            for (int c = 0; c < n_chunks; c++) {
                const int slot = c % kIxSlots, tb = c & 1;
                if (!tc::mbar_wait(bar(kBarStConv + slot), (c / kIxSlots) & 1, kIxWaitLimit)) ok = false;
                if (c >= 2 && !tc::mbar_wait(bar(kBarAccEmpty + tb), ((c >> 1) - 1) & 1, kIxWaitLimit)) ok = false;
                tc::fence_after_sync();
                const uint32_t d = tmem + tb * 32;
                const uint32_t t0 = slots_addr + slot * kIxSlotBytes + (kQ8 ? kIxTermBytes : 0);
#pragma unroll
                for (int ks = 0; ks < kIdxDim / 16; ks++) {
                    const uint32_t a = t0 + (ks >> 2) * (kQ8 ? kIxAtomBytes : 2 * kIxAtomBytes) + (ks & 3) * 32;
                    tc::mma_bf16(d, tc::desc_sw128(a, 1024), tc::desc(q_addr + ks * 256, 128, 2048), idesc,
                                 ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(bar(kBarStEmpty + slot));
                tc::mma_commit(bar(kBarAccFull + tb));
            }
            GLM_TL_AT(glm_tl_index, 2, 32);
        }
    } else if (warp == 2) {
        // ---------------- the multi-CTA selection's sample threshold ----------------
        // Once the epilogue has scored the sample chunks: publish this CTA's largest sample keys,
        // meet the query's other CTAs, and select the threshold from all published keys.
        if (sample) {
            unsigned *cq = sel.counters + static_cast<int64_t>(n) * kCntWords;
            if (sel.early) asm volatile("griddepcontrol.wait;" ::: "memory");   // the meeting word is zeroed
            bool waited = tc::mbar_wait(bar(kBarSample), 0, kIxWaitLimit);   // the sample keys are written
            __syncwarp();
            GLM_TL_AT(glm_tl_index, 13, 64);
            const unsigned thr = sample_threshold(samp, min(s0, hi - lo), r_pub, static_cast<unsigned>(k_s),
                                                  sel.gsamp + static_cast<int64_t>(n) * kSampleUnion, g,
                                                  &cq[kCntSample], g_eff, scr, waited);
            GLM_TL_AT(glm_tl_index, 5, 64);
            if (lane == 0) {
                flag[kFlThr] = thr;
                if (!waited) flag[kFlWait] = 1;
            }
            __syncwarp();
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------- epilogue: TMEM lane quadrant (warp % 4) ----------------
        // fp32 keys: quadrants 0-1 hold the hi dots of pools 32 q + lane, quadrants 2-3 the lo dots
        // of pools 32 (q - 2) + lane, handed over through the exchange buffer ([head][pool]: lanes
        // write consecutive words). int8 keys: rows 16 q + lane (lanes 0-15) of an M = 64 tile.
        const int qd = warp & 3;
        const int n_st = min(n_st0, n_chunks);   // chunks of the sample (multi-CTA selection)
        float *xch = reinterpret_cast<float *>(smem + IxLayout::kXch);
        const bool scorer = kQ8 || qd < 2;
        for (int c = 0; c < n_chunks; c++) {
            const int tb = c & 1;
            const int r = kQ8 ? qd * 16 + lane : (qd & 1) * 32 + lane;   // row of the chunk
            const bool has_row = kQ8 ? lane < 16 : true;
            const int p = lo + c * kIxTile + r;
            float ksc = 1.0f;   // the pool's int8 scale (loaded before the wait)
            if (kQ8 && has_row && p < hi) ksc = __ldg(key_scales + static_cast<int64_t>(b) * ld_pools + p);
            if (!tc::mbar_wait(bar(kBarAccFull + tb), (c >> 1) & 1, kIxWaitLimit)) ok = false;
            __syncwarp();
            tc::fence_after_sync();
            uint32_t rr[32];
            tc::tmem_ld32(tmem + (static_cast<uint32_t>(qd * 32) << 16) + tb * 32, rr);
            tc::tmem_wait_ld();
            float *xb = xch + tb * (kIxTile * kIdxHeads);
            if (!scorer) {   // lo dots: to the exchange buffer for the warp holding the same pools' hi dots
#pragma unroll
                for (int h2 = 0; h2 < kIdxHeads; h2++) xb[h2 * kIxTile + r] = __uint_as_float(rr[h2]);
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(kBarXch + tb));
            } else {
                if (!kQ8) {
                    if (!tc::mbar_wait(bar(kBarXch + tb), (c >> 1) & 1, kIxWaitLimit)) ok = false;
#pragma unroll
                    for (int h2 = 0; h2 < kIdxHeads; h2++)
                        rr[h2] = __float_as_uint(__uint_as_float(rr[h2]) + xb[h2 * kIxTile + r]);
                }
                uint32_t digit = 0xffffffffu;
                if (has_row && p < hi) {
                    float sc = 0.0f;
#pragma unroll
                    for (int h2 = 0; h2 < kIdxHeads; h2++) sc = fmaf(ws[h2], fmaxf(__uint_as_float(rr[h2]), 0.0f), sc);
                    // relu(s y) = s relu(y) for s > 0: the int8 scale, or the row's 2^-e_p (exact)
                    sc *= kQ8 ? ksc : ps_ring[(c % kIxPsDepth) * kIxTile + r];
                    srow[p] = sc;
                    if (keep_local) sloc[p - lo] = sc;
                    const uint32_t key = score_key(sc);
                    if (sample && c < n_st) samp[p - lo] = key;
                    digit = key >> (32 - kHistBitsTop);
                }
                if (select && !multi && digit != 0xffffffffu) atomicAdd(&hist[digit], 1u);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(kBarAccEmpty + tb));
            if (c == 0) GLM_TL_AT(glm_tl_index, 12, 128);
            if (scorer && sample && c == n_st - 1) {   // the sample keys of this warp's rows are written
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(kBarSample));
            }
        }
        GLM_TL_AT(glm_tl_index, 3, 128);
    } else if (warp >= 16 - kIxConv) {
        // ---------------- converters: rows 8 cw .. 8 cw + 7 of each chunk, in place ----------------
        const int cw = warp - (16 - kIxConv);
        for (int c = 0; c < n_chunks; c++) {
            const int slot = c % kIxSlots;
            const uint32_t ph = (c / kIxSlots) & 1;
            const int rows_c = min(kIxTile, hi - (lo + c * kIxTile));
            unsigned char *st = slots + slot * kIxSlotBytes;
            if (!tc::mbar_wait(bar(kBarStFull + slot), ph, kIxWaitLimit)) ok = false;
            if constexpr (kQ8) {   // four int8 codes -> four exact fp16, beside the codes in the slot
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int r = cw * 8 + i;
                    const uint32_t v = r < rows_c ? *reinterpret_cast<const uint32_t *>(st + r * kIdxDim + lane * 4) : 0u;
                    const int off = (lane >> 4) * kIxAtomBytes + r * 128 + ((((lane & 15) >> 1) ^ (r & 7)) << 4) + (lane & 1) * 8;
                    *reinterpret_cast<uint2 *>(st + kIxTermBytes + off) = codes_to_f16x4(v);
                }
            } else {
                float4 x[8];
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int r = cw * 8 + i;
                    x[i] = r < rows_c ? *reinterpret_cast<const float4 *>(st + r * (kIdxDim * 4) + lane * 16)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                // every warp has read its rows before any rewrites the slot
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(kBarStRead + slot));
                float m[8];
#pragma unroll
                for (int i = 0; i < 8; i++)
                    m[i] = fmaxf(fmaxf(fabsf(x[i].x), fabsf(x[i].y)), fmaxf(fabsf(x[i].z), fabsf(x[i].w)));
                const float mrow = butterfly<8, true>(m);   // lane l: max of row (l >> 2) & 7
                if (!tc::mbar_wait(bar(kBarStRead + slot), ph, kIxWaitLimit)) ok = false;
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int r = cw * 8 + i;
                    const int e = pow2_exponent(__shfl_sync(0xffffffffu, mrow, 4 * i));
                    const float f = pow2f(e);
                    const float4 y = make_float4(x[i].x * f, x[i].y * f, x[i].z * f, x[i].w * f);
                    const uint32_t h0 = f16x2_rn(y.x, y.y), h1 = f16x2_rn(y.z, y.w);
                    const uint32_t l0 = f16x2_rn(y.x - f16_lo_f(h0), y.y - f16_hi_f(h0));
                    const uint32_t l1 = f16x2_rn(y.z - f16_lo_f(h1), y.w - f16_hi_f(h1));
                    // K atom (lane / 16) holds the hi rows at +0 and the lo rows at +8 KB
                    const int off = (lane >> 4) * (2 * kIxAtomBytes) + r * 128 + ((((lane & 15) >> 1) ^ (r & 7)) << 4) + (lane & 1) * 8;
                    *reinterpret_cast<uint2 *>(st + off) = make_uint2(h0, h1);
                    *reinterpret_cast<uint2 *>(st + kIxAtomBytes + off) = make_uint2(l0, l1);
                    if (lane == i) ps_ring[(c % kIxPsDepth) * kIxTile + r] = pow2f(-e);
                }
            }
            tc::fence_proxy_async();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(kBarStConv + slot));
        }
        GLM_TL_AT(glm_tl_index, 4, 256);
    }
    if (!ok && status) atomicOr(status, 4);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 64);
    }
    }   // lo < hi
    if (sel.early) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    GLM_TL(glm_tl_index, 6);
    if (!select) return;
    const unsigned count = static_cast<unsigned>(min(sel.select_k, n_vis));
    auto score_at = [&](int i) { return keep_local ? sloc[i - lo] : __ldcg(srow + i); };

    // ---------------- phase 2: selection (every MMA and bulk copy of this CTA has completed) ----------------
    unsigned *cnt = sel.counters + static_cast<int64_t>(n) * kCntWords;
    if (multi) {
        if (lo >= hi) return;   // no score range: not part of the query's selection
        if (tid == 0 && flag[kFlWait] && status) atomicOr(status, 8);
        const unsigned thr = flag[kFlThr];   // the sample threshold (0: every score is a candidate)
        // this CTA's candidates (scores whose key reaches the sample threshold) go to the query's
        // list at an offset taken from its counter: count them, take the offset, write them
        unsigned long long *cand_q = sel.alist + static_cast<int64_t>(n) * sel.list_cap;   // holds n_vis
        unsigned mine = 0u;
#pragma unroll 1
        for (int b0 = lo; b0 < hi; b0 += kIxThreads) {
            const int i = b0 + tid;
            mine += static_cast<unsigned>(__syncthreads_count(i < hi && score_key(score_at(i)) >= thr));
        }
        if (tid == 0) {
            s.n_a = atomicAdd(&cnt[kCntTicket], mine);
            s.n_b = 0;
        }
        __syncthreads();
        const unsigned base = s.n_a;
        GLM_TL(glm_tl_index, 7);
#pragma unroll 1
        for (int b0 = lo; b0 < hi; b0 += kIxThreads) {
            const int i = b0 + tid;
            const uint32_t key = i < hi ? score_key(score_at(i)) : 0u;
            const bool take = i < hi && key >= thr;
            if (!__any_sync(0xffffffffu, take)) continue;
            const unsigned pos = warp_append(take, &s.n_b);
            if (take) {
                cand_q[base + pos] = compose(key, i);
                const long long t0 = pb + static_cast<long long>(kKpool) * i;   // warm L2 for the expansion
                if (sel.rows && sel.slot_map && t0 >= 0 && t0 + kKpool <= sel.ld_slot)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(sel.slot_map + static_cast<int64_t>(b) * sel.ld_slot + t0));
            }
        }
        __syncthreads();
        GLM_TL(glm_tl_index, 8);
        if (tid == 0) {   // release the candidates, wait (acquire) for every CTA's
            flag[kFlWait] = grid_barrier(&cnt[kCntArrive], g_eff) ? 0u : 1u;
            if (flag[kFlWait] && status) atomicOr(status, 8);
        }
        __syncthreads();
        if (flag[kFlWait]) return;   // gave up waiting: the status word reports it
        GLM_TL(glm_tl_index, 9);
        const unsigned total = __ldcg(&cnt[kCntTicket]);
        if (total < count || total > static_cast<unsigned>(kBoundCap)) {
            // the threshold let too few (or too many) through: CTA 0 selects exactly over every
            // score of the row and writes the outputs
            if (g != 0) return;
            auto get = [&](int i) { return compose(score_key(__ldcg(srow + i)), i); };
            radix_select(get, n_vis, count, 0, 0ull, s);
            collect_from(get, n_vis, ~0ull << (64 - s.done), s.prefix, 0u, s);
            sort_selected(s.cand, static_cast<int>(count), s);
            write_outputs(sel, n, b, valid_b, pb, seq_len, qp, count, s);
            return;
        }
        // every CTA: all candidates on chip, then the rank of its share of them -- the number of
        // larger composites (they are unique) -- and, for the count best, their outputs
#pragma unroll 1
        for (unsigned i = tid; i < total; i += kIxThreads) s.bnd[i] = __ldcg(cand_q + i);
        __syncthreads();
        GLM_TL(glm_tl_index, 10);
#pragma unroll 1
        for (unsigned j = static_cast<unsigned>(g + g_eff * warp); j < total; j += static_cast<unsigned>(g_eff * (kIxThreads / 32))) {
            const unsigned long long c = s.bnd[j];
            unsigned gt = 0u;
#pragma unroll 4
            for (unsigned i = lane; i < total; i += 32) gt += s.bnd[i] > c ? 1u : 0u;
            const unsigned r = __reduce_add_sync(0xffffffffu, gt);
            if (r < count) write_ranked(sel, n, b, pb, r, id_of(c), lane);
        }
        if (g == 0) write_unranked(sel, n, b, pb, seq_len, qp, count);
        GLM_TL(glm_tl_index, 11);
        return;
    }
    // one CTA: lo = 0, hi = n_vis, the histogram and the scores on chip
    int bstar = -1;   // every visible pool is selected
    if (n_vis > sel.select_k) {
        block_find_bin(hist, static_cast<unsigned>(sel.select_k), s);
        bstar = static_cast<int>(s.bin);
    }
    if (tid == 0) { s.n_a = 0; s.n_b = 0; }
    for (int i = tid; i < kHistBins; i += kIxThreads) s.hist2[i] = 0;
    __syncthreads();
    classify_range(score_at, lo, hi, bstar, s.hist2, s);
    __syncthreads();
    if (sel.rows && sel.slot_map) {   // warm L2 with the slot-map lines the expansion may read
        const unsigned la = min(s.n_a, static_cast<unsigned>(kMaxSelect));
        const unsigned lb = min(s.n_b, static_cast<unsigned>(kBoundCap));
        for (unsigned i = tid; i < la + lb; i += kIxThreads) {
            const int p = id_of(i < la ? s.cand[i] : s.bnd[i - la]);
            const long long t0 = pb + static_cast<long long>(kKpool) * p;
            if (t0 >= 0 && t0 + kKpool <= sel.ld_slot)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(sel.slot_map + static_cast<int64_t>(b) * sel.ld_slot + t0));
        }
    }
    const unsigned nA = min(s.n_a, static_cast<unsigned>(kMaxSelect));
    const unsigned nB = s.n_b;
    const bool b_complete = nB <= static_cast<unsigned>(kBoundCap);
    const unsigned long long top = static_cast<unsigned long long>(bstar < 0 ? 0 : bstar);
    auto get_b = [&](int i) -> unsigned long long {   // list B straight from the scores
        const uint32_t key = score_key(__ldcg(srow + i));
        return (key >> (32 - kHistBitsTop)) == top ? compose(key, i) : 0ull;
    };
    finish_selection(count, nA, nB, b_complete, bstar, s.hist2, get_b, n_vis, s);
    write_outputs(sel, n, b, valid_b, pb, seq_len, qp, count, s);
}

cudaError_t set_cross_cta_wait_limit(uint32_t polls) {
    return cudaMemcpyToSymbol(g_cross_cta_wait_limit, &polls, sizeof(polls));
}

int index_select_ctas(int n_q, int64_t ld_pools, int num_sms) {
    int G = num_sms / n_q;   // every CTA resident at once (one per SM): the selection's grid barrier
    if (G < 1) G = 1;
    const int64_t max_tiles = (ld_pools + kIxTile - 1) / kIxTile;
    if (G > max_tiles) G = static_cast<int>(max_tiles > 0 ? max_tiles : 1);
    return G;
}

cudaError_t launch_index_select_tc(const void *q_idx, const float *w, const void *keys,
                                   const float *key_scales, int64_t ld_pools, const int32_t *q_seq,
                                   const int32_t *q_pos, const int32_t *pad, const int32_t *len, int batch,
                                   int n_q, float *scores, bool fill_invisible, const IxSelectArgs &sel,
                                   int *status, int num_sms, cudaStream_t stream) {
    const int G = index_select_ctas(n_q, ld_pools, num_sms);
    const int smem = IxLayout::kAlloc;
    auto kernel = key_scales ? index_select_tc_kernel<true> : index_select_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // No cooperative attribute: a cooperative grid cannot start under programmatic dependent launch
    // before its predecessor ends, which would forfeit the early streaming. Co-residency of the
    // grid barrier's CTAs holds by construction: G * n_q <= the SM count at one CTA per SM (the
    // shared memory allows no second), and a later kernel of the stream can only launch once every
    // CTA of this one has started. The wait is bounded and reports through the status word.
    e = launch_pdl(kernel, dim3(G, n_q), dim3(kIxThreads), smem, stream, static_cast<const uint16_t *>(q_idx), w,
                   keys, key_scales, ld_pools, q_seq, q_pos, pad, len, batch, scores, fill_invisible ? 1 : 0, sel,
                   status);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace glm
