// index_gemm.cu -- relu head-weighted index scores of many queries at once (a prefill chunk: its
// queries share their sequence's pooled keys) on the sm_100a tensor cores
// ("Module glm5next_dsa_ref": index_scores -- matmul -> relu -> head-weighted sum --; "GLM-5.3-Flash"
// pypto-lib page, 'Checkpoint shape': indexer 32 heads x 128):
//     score[n][p] = sum_h w[n][h] * max(0, sum_d q_idx[n][h][d] * pooled[b][p][d])
//
// The pooled keys are the MMA M dimension and four queries' 32 heads the N dimension, so that a
// tile of 256 pooled keys, converted once, serves every query of its sequence:
//   1. index_qprep_kernel: each (query, head) as fp16 scaled by the power of two 2^e that puts its
//      largest magnitude in [2^14, 2^15) (exact for every bf16 value down to 2^-31 of that
//      largest) with w' = w 2^-e, and each query's visible pool count and sequence; padded with
//      zeros to a multiple of 4 queries;
//   2. index_gemm_kernel, grid (tiles of 256 pools, query splits, sequences), 12 warps:
//      * warps 4-11 read the tile's fp32 keys (two bulk copies) and rewrite each half of 128 pools
//        in place as two fp16 terms per value after a per-pool power of two (hi = rn(x 2^e_p),
//        lo = rn(x 2^e_p - hi): together x to 2^-22 of the pool's largest), in the 128-byte
//        swizzle K-major layout;
//      * warp 0 streams each group of 4 queries' fp16 query block (128 rows x 128 dims, two TMA
//        boxes, 128-byte swizzle) through a ring of 2 and their w' through a ring of 4;
//      * warp 1 issues per group and half 16 UMMAs (M = 128 pools, N = 128 = 4 queries x 32
//        heads, K = 16; the hi term's 8 K steps, then the lo term's) into one of two fp32
//        accumulators in tensor memory (2 x 128 columns each);
//      * warps 4-11 (TMEM lane quadrant warp % 4, half (warp - 4) / 4) read the accumulator, apply
//        relu, w' and 2^-e_p, and write the scores (-inf past the query's visible pools).
//   A group with no query of the CTA's sequence is skipped; one whose queries see none of the
//   tile's pools gets its -inf scores without the MMAs.
// The work is 2 x 2 x 128 x 32 FLOP per (query, pool) on the tensor cores; each converted key tile
// is reused by every query, and each query block (re-read from L2) by 256 pools.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace glm {

GLM_TL_TABLE(glm_tl_gemm)

constexpr int kGmThreads = 384;
constexpr int kGmHalf = 128;                           // pools per UMMA (M)
constexpr int kGmTile = 2 * kGmHalf;                   // pools per CTA
constexpr int kGmGroup = 4;                            // queries per UMMA N (4 x 32 heads = 128)
constexpr int kGmN = kGmGroup * kIdxHeads;             // 128
constexpr int kGmAtom = kGmHalf * 128;                 // 16 KB: one 64-dim K atom of one fp16 term of one half
constexpr int kGmQBox = kGmN * 128;                    // 16 KB: one 64-dim K atom of a group's queries
constexpr int kGmQSlots = 2;
constexpr int kGmWSlots = 4;
constexpr uint32_t kGmWaitLimit = 1u << 22;

// mbarriers
constexpr int kGbRaw = 0;        // [2] a half's fp32 keys have landed (tx)
constexpr int kGbRead = 2;       // every converter warp holds its rows of a half in registers (8 arrivals, twice)
constexpr int kGbA = 3;          // the fp16 terms of both halves are written (8 arrivals)
constexpr int kGbQFull = 4;      // [2] query block landed (tx)
constexpr int kGbQEmpty = 6;     // [2] query block read by the MMAs (commit)
constexpr int kGbDFull = 8;      // [2] accumulator ready (commit)
constexpr int kGbDEmpty = 10;    // [2] accumulator read (8 epilogue warps)
constexpr int kGbWFull = 12;     // [4] w' landed (tx)
constexpr int kGbWEmpty = 16;    // [4] w' read (8 epilogue warps)
constexpr int kGbCount = kGbWEmpty + kGmWSlots;

struct GmLayout {                                      // offsets from a 1024-byte aligned base
    static constexpr int kA = 0;                                      // 128 KB: fp32 keys, then [half][term][atom]
    static constexpr int kQ = kA + 8 * kGmAtom;                       // [2][32 KB] query blocks
    static constexpr int kW = kQ + kGmQSlots * 2 * kGmQBox;           // [4][4 queries][32] fp32 w'
    static constexpr int kPs = kW + kGmWSlots * kGmGroup * kIdxHeads * 4;   // [256] fp32 2^-e_p
    static constexpr int kBar = kPs + kGmTile * 4;
    static constexpr int kTmem = kBar + kGbCount * 8;
    static constexpr int kBytes = kTmem + 16;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(GmLayout::kAlloc <= 232448, "shared memory of one CTA");
static_assert(2 * kGmQSlots * kGmN <= 512, "two accumulators of two halves in 512 TMEM columns");

__device__ __forceinline__ uint32_t gm_f16x2(float a, float b) {   // .x = a (low half)
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}
__device__ __forceinline__ float gm_lo(uint32_t p) { return __half2float(__ushort_as_half(static_cast<unsigned short>(p & 0xffffu))); }
__device__ __forceinline__ float gm_hi(uint32_t p) { return __half2float(__ushort_as_half(static_cast<unsigned short>(p >> 16))); }
// The exponent e that puts a nonzero magnitude m in [2^14, 2^15) once scaled by 2^e (clamped so
// that 2^e and 2^-e are normal floats); 0 for m = 0.
__device__ __forceinline__ int gm_exponent(float m) {
    if (!(m > 0.0f)) return 0;
    const int E = static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127;
    return min(120, max(-120, 14 - E));
}
__device__ __forceinline__ float gm_pow2(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// What a CTA of sequence b and tile start p0 does with group g: 0 nothing (no query of b), 1 only
// -inf scores (no query of b sees a pool of the tile), 2 the MMAs. meta: (visible pools,
// sequence) per query, sequence -1 for the padding.
__device__ __forceinline__ int gm_kind(const int2 *meta, int g, int b, int64_t p0) {
    const int4 *m4 = reinterpret_cast<const int4 *>(meta + static_cast<int64_t>(g) * kGmGroup);
    int k = 0;
#pragma unroll
    for (int h = 0; h < kGmGroup / 2; h++) {
        const int4 v = m4[h];
        if (v.y == b) k = max(k, v.x > p0 ? 2 : 1);
        if (v.w == b) k = max(k, v.z > p0 ? 2 : 1);
    }
    return k;
}

// ------------------------------------------------------------------------------------------------
// 1. query preparation: one CTA of 128 threads per (padded) query; thread t holds head t / 4,
//    dims 32 (t % 4) .. + 31. A query of no valid sequence gets (0 visible pools, sequence 0):
//    every score of its row -inf.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) index_qprep_kernel(const uint16_t *__restrict__ q_idx,
                                                          const float *__restrict__ w, int n_q,
                                                          const int32_t *__restrict__ q_seq,
                                                          const int32_t *__restrict__ q_pos,
                                                          const int32_t *__restrict__ pad,
                                                          const int32_t *__restrict__ len, int batch,
                                                          int64_t ld_pools, uint16_t *__restrict__ q16,
                                                          float *__restrict__ wp, int2 *__restrict__ meta) {
    pdl_begin();
    const int n = blockIdx.x, t = threadIdx.x, h = t >> 2, part = t & 3;
    uint4 *dst = reinterpret_cast<uint4 *>(q16 + (static_cast<int64_t>(n) * kIdxHeads + h) * kIdxDim + part * 32);
    if (n >= n_q) {   // padding of the last group
#pragma unroll
        for (int i = 0; i < 4; i++) dst[i] = make_uint4(0u, 0u, 0u, 0u);
        if (part == 0) wp[static_cast<int64_t>(n) * kIdxHeads + h] = 0.0f;
        if (t == 0) meta[n] = make_int2(0, -1);
        return;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(q_idx + (static_cast<int64_t>(n) * kIdxHeads + h) * kIdxDim + part * 32);
    uint4 v[4];
    unsigned mb = 0u;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        v[i] = __ldg(src + i);
        const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 4; e++) mb = max(mb, max(w4[e] & 0x7fffu, (w4[e] >> 16) & 0x7fffu));
    }
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
    const int f = gm_exponent(__uint_as_float(mb << 16));
    const float sc = gm_pow2(f);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; e++) o[e] = gm_f16x2(__uint_as_float(w4[e] << 16) * sc, __uint_as_float(w4[e] & 0xffff0000u) * sc);
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (part == 0) wp[static_cast<int64_t>(n) * kIdxHeads + h] = __ldg(w + static_cast<int64_t>(n) * kIdxHeads + h) * gm_pow2(-f);
    if (t == 0) {
        const int b = q_seq[n];
        const bool ok = b >= 0 && b < batch;
        meta[n] = make_int2(ok ? visible_pools(pad[b], len[b], q_pos[n], ld_pools) : 0, ok ? b : 0);
    }
}

// ------------------------------------------------------------------------------------------------
// 2. the scores
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kGmThreads, 1) index_gemm_kernel(
    const __grid_constant__ CUtensorMap map_q, const float *__restrict__ wp, const int2 *__restrict__ meta,
    const float *__restrict__ pooled, int64_t ld_pools, int n_groups, int groups_per_split,
    float *__restrict__ scores, int *__restrict__ status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z;
    const int64_t p0 = static_cast<int64_t>(blockIdx.x) * kGmTile;
    const int rows_valid = static_cast<int>(ld_pools - p0 < kGmTile ? ld_pools - p0 : static_cast<int64_t>(kGmTile));
    const int g0 = blockIdx.y * groups_per_split, g1 = min(n_groups, g0 + groups_per_split);
    const uint32_t bar0 = tc::smem_addr(smem + GmLayout::kBar);
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + GmLayout::kTmem);
    float *ps = reinterpret_cast<float *>(smem + GmLayout::kPs);
    const uint32_t sa = tc::smem_addr(smem + GmLayout::kA), sq = tc::smem_addr(smem + GmLayout::kQ);
    GLM_TL(glm_tl_gemm, 0);

    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), 512);
        tc::tmem_relinquish();
        tc::fence_before_sync();
    }
    if (tid == 32) {
        tc::mbar_init(bar(kGbRaw), 1);
        tc::mbar_init(bar(kGbRaw + 1), 1);
        tc::mbar_init(bar(kGbRead), 8);
        tc::mbar_init(bar(kGbA), 8);
        for (int s = 0; s < kGmQSlots; s++) {
            tc::mbar_init(bar(kGbQFull + s), 1);
            tc::mbar_init(bar(kGbQEmpty + s), 1);
            tc::mbar_init(bar(kGbDFull + s), 1);
            tc::mbar_init(bar(kGbDEmpty + s), 8);
        }
        for (int s = 0; s < kGmWSlots; s++) {
            tc::mbar_init(bar(kGbWFull + s), 1);
            tc::mbar_init(bar(kGbWEmpty + s), 8);
        }
        tc::mbar_fence_init();
    }
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // the query blocks, w' and meta are written by the preceding kernel
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // a wait that gives up marks the thread; it then skips its later waits (the outputs are
    // invalid and the status word says so), so that a broken pipeline ends within one wait limit
    bool ok = true;
    auto wait = [&](int i, uint32_t parity) {
        if (ok && !tc::mbar_wait(bar(i), parity, kGmWaitLimit)) ok = false;
    };

    if (warp == 0) {
        if (lane == 0) {
            // the tile's fp32 keys (one contiguous copy per half), then the query groups through the rings
            asm volatile("fence.proxy.async.global;" ::: "memory");
            for (int t = 0; t < 2; t++) {
                const int rows = min(kGmHalf, max(0, rows_valid - t * kGmHalf));
                if (rows > 0) {
                    tc::mbar_arrive_expect_tx(bar(kGbRaw + t), static_cast<uint32_t>(rows) * kIdxDim * 4);
                    tc::bulk_g2s(sa + t * 4 * kGmAtom, pooled + (static_cast<int64_t>(b) * ld_pools + p0 + t * kGmHalf) * kIdxDim,
                                 static_cast<uint32_t>(rows) * kIdxDim * 4, bar(kGbRaw + t));
                } else {
                    tc::mbar_arrive(bar(kGbRaw + t));
                }
            }
            for (int g = g0, i = 0; g < g1; g++) {
                if (gm_kind(meta, g, b, p0) != 2) continue;
                const int sqs = i % kGmQSlots, sws = i % kGmWSlots;
                if (i >= kGmWSlots) wait(kGbWEmpty + sws, ((i / kGmWSlots) - 1) & 1);
                tc::mbar_arrive_expect_tx(bar(kGbWFull + sws), kGmGroup * kIdxHeads * 4);
                tc::bulk_g2s(tc::smem_addr(smem + GmLayout::kW) + sws * kGmGroup * kIdxHeads * 4,
                             wp + static_cast<int64_t>(g) * kGmGroup * kIdxHeads, kGmGroup * kIdxHeads * 4, bar(kGbWFull + sws));
                if (i >= kGmQSlots) wait(kGbQEmpty + sqs, ((i / kGmQSlots) - 1) & 1);
                tc::mbar_arrive_expect_tx(bar(kGbQFull + sqs), 2 * kGmQBox);
                for (int a = 0; a < 2; a++)
                    tc::tma_load_2d(sq + sqs * 2 * kGmQBox + a * kGmQBox, &map_q, bar(kGbQFull + sqs), a * 64, g * kGmN);
                i++;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer: per group and half, 8 K steps of the hi term, then 8 of the lo term
            const uint32_t idesc = tc::idesc_f16(kGmHalf, kGmN, false, false);
            wait(kGbA, 0);
            tc::fence_after_sync();
            for (int g = g0, i = 0; g < g1; g++) {
                if (gm_kind(meta, g, b, p0) != 2) continue;
                const int s = i % kGmQSlots;
                wait(kGbQFull + s, (i / kGmQSlots) & 1);
                if (i >= kGmQSlots) wait(kGbDEmpty + s, ((i / kGmQSlots) - 1) & 1);
                tc::fence_after_sync();
                const uint32_t qb = sq + s * 2 * kGmQBox;
#pragma unroll
                for (int t = 0; t < 2; t++) {
                    const uint32_t d = tmem + s * 2 * kGmN + t * kGmN;
#pragma unroll
                    for (int term = 0; term < 2; term++) {
#pragma unroll
                        for (int ks = 0; ks < kIdxDim / 16; ks++) {
                            const uint32_t a = sa + ((t * 2 + term) * 2 + (ks >> 2)) * kGmAtom + (ks & 3) * 32;
                            const uint32_t bq = qb + (ks >> 2) * kGmQBox + (ks & 3) * 32;
                            tc::mma_bf16(d, tc::desc_sw128(a, 1024), tc::desc_sw128(bq, 1024), idesc,
                                         (term > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                }
                tc::mma_commit(bar(kGbQEmpty + s));
                tc::mma_commit(bar(kGbDFull + s));
                i++;
            }
        }
    } else if (warp >= 4) {
        // ---- the keys, half by half: rows 16 cw .. 16 cw + 15 of the half, lane l holding dims 4 l .. 4 l + 3 ----
        const int cw = warp - 4;
        for (int t = 0; t < 2; t++) {
            wait(kGbRaw + t, 0);
            ok = __all_sync(0xffffffffu, ok);
            unsigned char *half = smem + GmLayout::kA + t * 4 * kGmAtom;
            float4 x[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const int r = cw * 16 + i;
                x[i] = t * kGmHalf + r < rows_valid ? *reinterpret_cast<const float4 *>(half + r * kIdxDim * 4 + lane * 16)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(kGbRead));
            wait(kGbRead, t);   // every row of the half read: rewrite in place
            ok = __all_sync(0xffffffffu, ok);
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const int r = cw * 16 + i;
                const float m = fmaxf(fmaxf(fabsf(x[i].x), fabsf(x[i].y)), fmaxf(fabsf(x[i].z), fabsf(x[i].w)));
                const int e = gm_exponent(__uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m))));
                const float f = gm_pow2(e);
                const float4 y = make_float4(x[i].x * f, x[i].y * f, x[i].z * f, x[i].w * f);
                const uint32_t h0 = gm_f16x2(y.x, y.y), h1 = gm_f16x2(y.z, y.w);
                const uint32_t l0 = gm_f16x2(y.x - gm_lo(h0), y.y - gm_hi(h0));
                const uint32_t l1 = gm_f16x2(y.z - gm_lo(h1), y.w - gm_hi(h1));
                // atom lane / 16 (dims 64 a ..), 16-byte chunk ((lane & 15) >> 1) ^ (r & 7), half lane & 1
                const int off = (lane >> 4) * kGmAtom + r * 128 + ((((lane & 15) >> 1) ^ (r & 7)) << 4) + (lane & 1) * 8;
                *reinterpret_cast<uint2 *>(half + off) = make_uint2(h0, h1);
                *reinterpret_cast<uint2 *>(half + 2 * kGmAtom + off) = make_uint2(l0, l1);
                if (lane == 0) ps[t * kGmHalf + r] = gm_pow2(-e);
            }
        }
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(kGbA));

        // ---- epilogue: TMEM lane quadrant warp % 4 of half (warp - 4) / 4: pool 128 t + 32 quad + lane ----
        const int quad = warp & 3, t = (warp - 4) >> 2;
        const int pr = t * kGmHalf + quad * 32 + lane;
        const int64_t p = p0 + pr;
        wait(kGbA, 0);   // (ps of every row written)
        ok = __all_sync(0xffffffffu, ok);
        const float psr = ps[pr];
        for (int g = g0, i = 0; g < g1; g++) {
            const int kind = gm_kind(meta, g, b, p0);
            if (kind == 0) continue;
            if (kind == 1) {
                for (int j = 0; j < kGmGroup; j++) {
                    const int64_t n = static_cast<int64_t>(g) * kGmGroup + j;
                    if (meta[n].y == b && p < ld_pools) scores[n * ld_pools + p] = -INFINITY;
                }
                continue;
            }
            const int s = i % kGmQSlots, sws = i % kGmWSlots;
            wait(kGbDFull + s, (i / kGmQSlots) & 1);
            wait(kGbWFull + sws, (i / kGmWSlots) & 1);
            ok = __all_sync(0xffffffffu, ok);   // the warp's TMEM loads below stay convergent
            __syncwarp();
            tc::fence_after_sync();
            const float *wq = reinterpret_cast<const float *>(smem + GmLayout::kW) + sws * kGmGroup * kIdxHeads;
#pragma unroll 1
            for (int j = 0; j < kGmGroup; j++) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + s * 2 * kGmN + t * kGmN + j * kIdxHeads, r);
                tc::tmem_wait_ld();
                const int64_t n = static_cast<int64_t>(g) * kGmGroup + j;
                const int2 m = meta[n];   // (visible pools, sequence; -1: padding)
                if (m.y != b || p >= ld_pools) continue;
                float sc = 0.0f;
#pragma unroll
                for (int h = 0; h < kIdxHeads; h++) sc = fmaf(wq[j * kIdxHeads + h], fmaxf(__uint_as_float(r[h]), 0.0f), sc);
                scores[n * ld_pools + p] = p < m.x ? sc * psr : -INFINITY;
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(bar(kGbDEmpty + s));
                tc::mbar_arrive(bar(kGbWEmpty + sws));
            }
            i++;
        }
    }
    if (!ok && status) atomicOr(status, 16);
    tc::fence_before_sync();
    __syncthreads();
    GLM_TL(glm_tl_gemm, 1);
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

size_t index_gemm_scratch_bytes(int n_q) {
    const size_t n_pad = static_cast<size_t>((n_q + kGmGroup - 1) / kGmGroup) * kGmGroup;
    const auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    return al(n_pad * kIdxHeads * kIdxDim * 2) + al(n_pad * kIdxHeads * 4) + al(n_pad * 8);
}

cudaError_t launch_index_gemm(const void *q_idx, const float *w, const float *pooled, int64_t ld_pools,
                              const int32_t *q_seq, const int32_t *q_pos, const int32_t *pad, const int32_t *len,
                              int batch, int n_q, float *scores, void *scratch, int *status, int num_sms,
                              cudaStream_t stream) {
    if (n_q <= 0 || ld_pools <= 0 || batch <= 0) return cudaSuccess;
    const int n_groups = (n_q + kGmGroup - 1) / kGmGroup;
    const size_t n_pad = static_cast<size_t>(n_groups) * kGmGroup;
    const auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    char *sp = static_cast<char *>(scratch);
    uint16_t *q16 = reinterpret_cast<uint16_t *>(sp);
    float *wp = reinterpret_cast<float *>(sp + al(n_pad * kIdxHeads * kIdxDim * 2));
    int2 *meta = reinterpret_cast<int2 *>(sp + al(n_pad * kIdxHeads * kIdxDim * 2) + al(n_pad * kIdxHeads * 4));
    cudaError_t e = launch_pdl(index_qprep_kernel, dim3(static_cast<unsigned>(n_pad)), dim3(128), 0, stream,
                               static_cast<const uint16_t *>(q_idx), w, n_q, q_seq, q_pos, pad, len, batch, ld_pools,
                               q16, wp, meta);
    if (e != cudaSuccess) return e;
    auto encode = tc::tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    // q16 fp16 [n_pad * 32 rows][128 dims]: boxes of 64 dims x 128 rows (one group), 128-byte swizzle
    CUtensorMap map_q;
    const cuuint64_t dim[2] = {static_cast<cuuint64_t>(kIdxDim), static_cast<cuuint64_t>(n_pad * kIdxHeads)};
    const cuuint64_t stride[1] = {static_cast<cuuint64_t>(kIdxDim) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kGmN)}, one[2] = {1, 1};
    CUresult r = encode(&map_q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, q16, dim, stride, box, one,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int tiles = static_cast<int>((ld_pools + kGmTile - 1) / kGmTile);
    // query splits (runs of whole groups): the count that minimises waves x (groups per CTA + the
    // key conversion, worth about 3 groups), at most 32 waves
    const int64_t units = static_cast<int64_t>(tiles) * batch;
    int gps = n_groups;
    int64_t best = -1;
    for (int s = 1; s <= n_groups; s++) {
        const int per = (n_groups + s - 1) / s;
        const int64_t splits_s = (n_groups + per - 1) / per;
        const int64_t waves = (units * splits_s + num_sms - 1) / num_sms;
        if (waves > 32 && best >= 0) break;
        const int64_t cost = waves * (per + 3);
        if (best < 0 || cost < best) { best = cost; gps = per; }
    }
    const int splits = (n_groups + gps - 1) / gps;
    const int smem = GmLayout::kAlloc;
    e = cudaFuncSetAttribute(index_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(index_gemm_kernel, dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(splits),
                                           static_cast<unsigned>(batch)),
                   dim3(kGmThreads), smem, stream, map_q, wp, meta, pooled, ld_pools, n_groups, gps, scores, status);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace glm
