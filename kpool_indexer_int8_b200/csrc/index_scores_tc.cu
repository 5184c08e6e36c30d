// index_scores_tc.cu -- relu head-weighted index scores on the sm_100a tensor cores
// ("Module glm5next_dsa_ref", index_scores: the matmul -> relu -> head-weighted sum chain;
// "GLM-5.3-Flash" pypto-lib page, 'Checkpoint shape': indexer 32 heads x 128):
//     score[n][p] = sum_h w[n][h] * max(0, sum_d q_idx[n][h][d] * pooled[b][p][d])
//
// Decode form: grid (G, n_q), G ~ SMs / n_q; CTA g of query n owns a contiguous range of the
// query's visible pools and walks it in tiles of 128 pools:
//   * the fp32 pooled keys of a tile (64 KB) are read straight into registers, one tile ahead of
//     the tensor cores (each warp load covers 8 pools x 128 contiguous bytes);
//   * each fp32 value x is split exactly into three bf16 terms (hi = rn(x), mid = rn(x - hi),
//     lo = rn(x - hi - mid)) written as 8x8 core matrices into a double-buffered shared tile;
//   * per term, 8 UMMAs (M = 128 pools, N = 32 heads, K = 16) accumulate q . term into an fp32
//     tile of tensor memory (double-buffered, 2 x 32 columns): with bf16 q exact, the three terms
//     reproduce q . x to fp32 accumulation accuracy;
//   * the epilogue (one TMEM lane = one pool per thread) applies relu and the head weights,
//     writes the score and adds its top-11-bit key digit to the selection histogram.
// HBM-bound: 512 bytes of pooled key per pool; the tensor cores run at a few percent.
#include "common.cuh"
#include "tc.cuh"
#include "topk.cuh"

namespace glm {

constexpr int kIxThreads = 256;
constexpr int kIxTile = 128;                       // pools per tile (UMMA M)
constexpr int kIxTermBytes = kIxTile * kIdxDim * 2; // one bf16 term of a tile: 32 KB
constexpr uint32_t kIxWaitLimit = 1u << 22;

struct IxLayout {
    static constexpr int kA = 0;                                  // [2 buffers][3 terms][32 KB]
    static constexpr int kQ = kA + 2 * 3 * kIxTermBytes;          // 32 heads x 128 dims bf16 (8 KB)
    static constexpr int kHist = kQ + kIdxHeads * kIdxDim * 2;    // 2048 uint32
    static constexpr int kW = kHist + kHistBins * 4;              // 32 fp32 head weights
    static constexpr int kBar = kW + kIdxHeads * 4;               // 2 mbarriers
    static constexpr int kTmem = kBar + 16;
    static constexpr int kBytes = kTmem + 16;
};

__device__ __forceinline__ uint32_t bf16_pair(float a, float b) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(a))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(b))) << 16);
}
__device__ __forceinline__ float bf16_lo_f(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t p) { return __uint_as_float(p & 0xffff0000u); }

__device__ __forceinline__ float4 ld_stream(const float *p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(kIxThreads, 1) index_scores_tc_kernel(
    const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
    const float *__restrict__ pooled, int64_t ld_pools, const int32_t *__restrict__ q_seq,
    const int32_t *__restrict__ q_pos, const int32_t *__restrict__ pad,
    const int32_t *__restrict__ len, int batch, float *__restrict__ scores,
    unsigned *__restrict__ ghist, int fill_invisible, int *__restrict__ status) {
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *A = smem + IxLayout::kA;
    unsigned char *Qs = smem + IxLayout::kQ;
    unsigned *hist = reinterpret_cast<unsigned *>(smem + IxLayout::kHist);
    float *ws = reinterpret_cast<float *>(smem + IxLayout::kW);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + IxLayout::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + IxLayout::kTmem);

    const int n = blockIdx.y, g = blockIdx.x, G = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = q_seq[n];
    const int n_vis = (b >= 0 && b < batch) ? visible_pools(pad[b], len[b], q_pos[n], ld_pools) : 0;
    float *srow = scores + static_cast<int64_t>(n) * ld_pools;

    if (fill_invisible) {  // entries past the visible pools are -inf (split over the CTAs)
        const int64_t rest = ld_pools - n_vis;
        const int64_t share = (rest + G - 1) / G;
        const int64_t f0 = n_vis + static_cast<int64_t>(g) * share;
        const int64_t f1 = min(f0 + share, ld_pools);
        for (int64_t i = f0 + tid; i < f1; i += kIxThreads) srow[i] = -INFINITY;
    }
    int per = (n_vis + G - 1) / G;
    if (per < kIxTile) per = kIxTile;
    const int lo = g * per;
    const int hi = min(n_vis, lo + per);
    if (lo >= hi) return;
    const int n_tiles = (hi - lo + kIxTile - 1) / kIxTile;

    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), 64);
        tc::tmem_relinquish();
        tc::fence_before_sync();
    }
    if (tid == 32) {
        tc::mbar_init(tc::smem_addr(&bar[0]), 1);
        tc::mbar_init(tc::smem_addr(&bar[1]), 1);
        tc::mbar_fence_init();
    }
    // query block (bf16 [32 x 128], core matrices: head group stride 2048 B, dim group 128 B)
    const uint16_t *qn = q_idx + static_cast<int64_t>(n) * kIdxHeads * kIdxDim;
    for (int i = tid; i < kIdxHeads * kIdxDim / 8; i += kIxThreads) {
        const int h = i >> 4, dg = i & 15;
        *reinterpret_cast<uint4 *>(Qs + (h >> 3) * 2048 + dg * 128 + (h & 7) * 16) =
            __ldg(reinterpret_cast<const uint4 *>(qn + h * kIdxDim) + dg);
    }
    if (tid < kIdxHeads) ws[tid] = w[static_cast<int64_t>(n) * kIdxHeads + tid];
    if (ghist)
        for (int i = tid; i < kHistBins; i += kIxThreads) hist[i] = 0;

    const float *prow = pooled + static_cast<int64_t>(b) * ld_pools * kIdxDim;
    // unit u = it * 8 + warp covers pool group u % 16 (8 pools) and dim quad u / 16 (32 dims)
    float4 v[8][2];
    auto load_tile = [&](int t) {
#pragma unroll
        for (int it = 0; it < 8; it++) {
            const int u = it * 8 + warp;
            const int p = lo + t * kIxTile + (u & 15) * 8 + (lane & 7);
            const int d0 = (u >> 4) * 32 + (lane >> 3) * 8;
            if (p < hi) {
                v[it][0] = ld_stream(prow + static_cast<int64_t>(p) * kIdxDim + d0);
                v[it][1] = ld_stream(prow + static_cast<int64_t>(p) * kIdxDim + d0 + 4);
            } else {
                v[it][0] = make_float4(0.f, 0.f, 0.f, 0.f);
                v[it][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    };
    auto store_tile = [&](int buf) {
        unsigned char *base = A + buf * 3 * kIxTermBytes;
#pragma unroll
        for (int it = 0; it < 8; it++) {
            const int u = it * 8 + warp;
            const int off = (u & 15) * 2048 + ((u >> 4) * 4 + (lane >> 3)) * 128 + (lane & 7) * 16;
            const float x[8] = {v[it][0].x, v[it][0].y, v[it][0].z, v[it][0].w,
                                v[it][1].x, v[it][1].y, v[it][1].z, v[it][1].w};
            uint32_t h[4], m[4], l[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                h[e] = bf16_pair(x[2 * e], x[2 * e + 1]);
                const float r0 = x[2 * e] - bf16_lo_f(h[e]), r1 = x[2 * e + 1] - bf16_hi_f(h[e]);
                m[e] = bf16_pair(r0, r1);
                l[e] = bf16_pair(r0 - bf16_lo_f(m[e]), r1 - bf16_hi_f(m[e]));
            }
            *reinterpret_cast<uint4 *>(base + off) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4 *>(base + kIxTermBytes + off) = make_uint4(m[0], m[1], m[2], m[3]);
            *reinterpret_cast<uint4 *>(base + 2 * kIxTermBytes + off) = make_uint4(l[0], l[1], l[2], l[3]);
        }
    };

    load_tile(0);
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t idesc = tc::idesc_bf16(kIxTile, kIdxHeads, false, false);
    const uint32_t a_addr = tc::smem_addr(A), q_addr = tc::smem_addr(Qs);
    bool ok = true;

    auto epilogue = [&](int t) {
        const int buf = t & 1;
        if (!tc::mbar_wait(tc::smem_addr(&bar[buf]), (t >> 1) & 1, kIxWaitLimit)) ok = false;
        __syncwarp();
        tc::fence_after_sync();
        uint32_t r[32];
        tc::tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + buf * 32, r);
        tc::tmem_wait_ld();
        const int p = lo + t * kIxTile + warp * 32 + lane;
        uint32_t digit = 0xffffffffu;
        if (p < hi) {
            float s = 0.0f;
#pragma unroll
            for (int h2 = 0; h2 < kIdxHeads; h2++) s = fmaf(ws[h2], fmaxf(__uint_as_float(r[h2]), 0.0f), s);
            srow[p] = s;
            digit = score_key(s) >> (32 - kHistBitsTop);
        }
        if (ghist) hist_add(hist, digit);
    };

    for (int t = 0; t < n_tiles; t++) {
        const int buf = t & 1;
        if (t >= 2) {  // the MMAs of tile t-2 have released this buffer
            if (!tc::mbar_wait(tc::smem_addr(&bar[buf]), ((t - 2) >> 1) & 1, kIxWaitLimit)) ok = false;
        }
        store_tile(buf);
        if (t + 1 < n_tiles) load_tile(t + 1);
        tc::fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t d = tmem + buf * 32;
#pragma unroll
            for (int term = 0; term < 3; term++) {
                const uint32_t ab = a_addr + (buf * 3 + term) * kIxTermBytes;
#pragma unroll
                for (int ks = 0; ks < kIdxDim / 16; ks++)
                    tc::mma_bf16(d, tc::desc(ab + ks * 256, 128, 2048), tc::desc(q_addr + ks * 256, 128, 2048),
                                 idesc, (term > 0 || ks > 0) ? 1u : 0u);
            }
            tc::mma_commit(tc::smem_addr(&bar[buf]));
        }
        if (t >= 1 && warp < 4) epilogue(t - 1);
    }
    if (warp < 4) epilogue(n_tiles - 1);
    if (!ok && status) atomicOr(status, 4);
    tc::fence_before_sync();
    __syncthreads();
    if (ghist) {
        unsigned *gh = ghist + static_cast<int64_t>(n) * kHistBins;
        for (int i = tid; i < kHistBins; i += kIxThreads)
            if (hist[i]) atomicAdd(&gh[i], hist[i]);
    }
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 64);
    }
}

cudaError_t launch_index_scores_tc(const void *q_idx, const float *w, const float *pooled,
                                   int64_t ld_pools, const int32_t *q_seq, const int32_t *q_pos,
                                   const int32_t *pad, const int32_t *len, int batch, int n_q,
                                   float *scores, unsigned *ghist, bool fill_invisible, int *status,
                                   int num_sms, cudaStream_t stream) {
    int G = (num_sms + n_q - 1) / n_q;
    if (G < 1) G = 1;
    const int64_t max_tiles = (ld_pools + kIxTile - 1) / kIxTile;
    if (G > max_tiles) G = static_cast<int>(max_tiles > 0 ? max_tiles : 1);
    const int smem = IxLayout::kBytes;
    cudaError_t e = cudaFuncSetAttribute(index_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(G, n_q);
    index_scores_tc_kernel<<<grid, kIxThreads, smem, stream>>>(
        static_cast<const uint16_t *>(q_idx), w, pooled, ld_pools, q_seq, q_pos, pad, len, batch,
        scores, ghist, fill_invisible ? 1 : 0, status);
    return cudaGetLastError();
}

}  // namespace glm
