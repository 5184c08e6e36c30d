// mla_combine.cu -- log-sum-exp merge of split-KV partial softmax states (the final combine of
// the split-KV decode named in "GLM-5.3 Kernels" README, 'Included': titan_mla ... split-KV).
//
//   M = max_c m_c,  L = sum_c l_c e^{m_c - M},  out = (sum_c e^{m_c - M} acc_c) / L,
//   lse = M + log L.
// Chunks with l = 0 (no valid entry) contribute nothing (their accumulators were never written).
#include "common.cuh"
#include "sparse_mla.cuh"

namespace glm {

GLM_TL_TABLE(glm_tl_combine)

constexpr int kCombineWarps = 4;
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kCombineDims = 128;                      // latent dims of one CTA (4 per lane)
constexpr int kCombineLoads = 12;                      // chunks per warp whose partials load at once
constexpr int kMaxCombineChunks = 1024;                // 65,536 entries / 64-entry chunks

__device__ __forceinline__ void fma4(float4 &a, float w, const float4 &v) {
    a.x = fmaf(w, v.x, a.x);
    a.y = fmaf(w, v.y, a.y);
    a.z = fmaf(w, v.z, a.z);
    a.w = fmaf(w, v.w, a.w);
}

// One CTA of 4 warps per (head, 128 of the 512 latent dims, query); lane l of warp w holds dims
// 4 l .. 4 l + 3 of the CTA's slice for chunks w, w + 4, ... Every warp first requests its chunks'
// partial accumulators (up to kCombineLoads at once) while warp 0 reads every chunk's (m, l) and
// writes the weights e^{m_c - M} to shared memory, so that one round trip to L2 serves both; the
// four warps' sums meet in shared memory. A chunk without a valid entry (l = 0) was never
// written: its accumulator is dropped, never multiplied.
__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(const float *__restrict__ part_acc,
                                                                      const float *__restrict__ part_ml,
                                                                      int n_heads, int n_chunks,
                                                                      uint16_t *__restrict__ out,
                                                                      float *__restrict__ out_f32,
                                                                      float *__restrict__ lse,
                                                                      const int *__restrict__ poison) {
    GLM_TL(glm_tl_combine, 0);
    GLM_TL_SMID(glm_tl_combine);
    pdl_begin();
    GLM_TL(glm_tl_combine, 1);
    __shared__ float4 part[kCombineWarps - 1][32];
    __shared__ float wts[kMaxCombineChunks];
    __shared__ float red[2];
    const int h = blockIdx.x >> 2, quarter = blockIdx.x & 3, n = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ob = (static_cast<int64_t>(n) * n_heads + h) * kLatent + quarter * kCombineDims + 4 * lane;
    if (poison && __ldcg(poison) != 0) {   // a split CTA gave up a wait: its partial is missing
        if (warp == 0) {
            const uint32_t nan2 = 0x7fc07fc0u;
            *reinterpret_cast<uint2 *>(out + ob) = make_uint2(nan2, nan2);
            if (out_f32) *reinterpret_cast<float4 *>(out_f32 + ob) = make_float4(__int_as_float(0x7fc00000),
                                                                                  __int_as_float(0x7fc00000),
                                                                                  __int_as_float(0x7fc00000),
                                                                                  __int_as_float(0x7fc00000));
            if (lse && quarter == 0 && lane == 0) lse[static_cast<int64_t>(n) * n_heads + h] = __int_as_float(0x7fc00000);
        }
        return;
    }
    const int64_t base = static_cast<int64_t>(n) * n_chunks * n_heads + h;   // (query, chunk 0, head)
    auto acc_at = [&](int c) {
        return __ldcg(reinterpret_cast<const float4 *>(part_acc + (base + static_cast<int64_t>(c) * n_heads) * kLatent +
                                                       quarter * kCombineDims) + lane);
    };
    auto ml_at = [&](int c) {
        return __ldcg(reinterpret_cast<const float2 *>(part_ml + 2 * (base + static_cast<int64_t>(c) * n_heads)));
    };
    float4 v[kCombineLoads];
#pragma unroll
    for (int u = 0; u < kCombineLoads; u++) {
        const int c = warp + u * kCombineWarps;
        v[u] = c < n_chunks ? acc_at(c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // warp 0: M over the chunks with an entry, the weights e^{m_c - M} (to shared memory) and L;
    // lane l keeps the pairs of chunks l and l + 32 in registers (more chunks are read again)
    if (warp == 0) {
        float2 keep[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const int c = lane + 32 * k;
            keep[k] = c < n_chunks ? ml_at(c) : make_float2(-INFINITY, 0.0f);
        }
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < 2; k++)
            if (keep[k].y > 0.0f) mx = fmaxf(mx, keep[k].x);
        for (int c = lane + 64; c < n_chunks; c += 32) {
            const float2 ml = ml_at(c);
            if (ml.y > 0.0f) mx = fmaxf(mx, ml.x);
        }
        mx = warp_max(mx);
        float Lp = 0.0f;
        for (int c = lane, k = 0; c < n_chunks; c += 32, k++) {
            const float2 ml = k < 2 ? keep[k < 2 ? k : 0] : ml_at(c);
            const float wc = ml.y > 0.0f ? expf(ml.x - mx) : 0.0f;
            wts[c] = wc;
            Lp = fmaf(ml.y, wc, Lp);
        }
        Lp = warp_sum(Lp);
        if (lane == 0) {
            red[0] = mx;
            red[1] = Lp;
        }
    }
    __syncthreads();
    const float mx = red[0], L = red[1];
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kCombineLoads; u++) {
        const int c = warp + u * kCombineWarps;
        if (c < n_chunks && wts[c] > 0.0f) fma4(a, wts[c], v[u]);
    }
    for (int c0 = warp + kCombineLoads * kCombineWarps; c0 < n_chunks; c0 += 8 * kCombineWarps) {
        float4 r[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int c = c0 + u * kCombineWarps;
            r[u] = (c < n_chunks && wts[c] > 0.0f) ? acc_at(c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int c = c0 + u * kCombineWarps;
            if (c < n_chunks && wts[c] > 0.0f) fma4(a, wts[c], r[u]);
        }
    }
    if (warp > 0) part[warp - 1][lane] = a;
    __syncthreads();
    if (warp > 0) return;
#pragma unroll
    for (int w2 = 0; w2 < kCombineWarps - 1; w2++) {
        const float4 b = part[w2][lane];
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const float o[4] = {a.x * inv, a.y * inv, a.z * inv, a.w * inv};
    const uint32_t lo = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[0]))) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[1]))) << 16);
    const uint32_t hi = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[2]))) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[3]))) << 16);
    *reinterpret_cast<uint2 *>(out + ob) = make_uint2(lo, hi);
    if (out_f32) *reinterpret_cast<float4 *>(out_f32 + ob) = make_float4(o[0], o[1], o[2], o[3]);
    if (lse && quarter == 0 && lane == 0) lse[static_cast<int64_t>(n) * n_heads + h] = L > 0.0f ? mx + logf(L) : -INFINITY;
    GLM_TL(glm_tl_combine, 2);
}

cudaError_t launch_mla_combine(const float *part_acc, const float *part_ml, int n_q, int n_heads,
                               int n_chunks, void *out, float *out_f32, float *lse,
                               cudaStream_t stream, const int *poison) {
    const dim3 grid(static_cast<unsigned>(n_heads * (kLatent / kCombineDims)), static_cast<unsigned>(n_q));
    launch_pdl(mla_combine_kernel, grid, dim3(kCombineThreads), 0, stream, part_acc, part_ml, n_heads, n_chunks,
               static_cast<uint16_t *>(out), out_f32, lse, poison);
    return cudaGetLastError();
}

}  // namespace glm

namespace glm {

// Log-sum-exp merge of attention results over disjoint sets of rows (context parallelism: each
// rank attends over the rows it holds; "the attention partials are merged by log-sum-exp in rank
// order", TensorFold issue #402, 'Credit'): with lse_r and the normalised out_r of part r,
//     LSE = log sum_r e^{lse_r},   out = sum_r e^{lse_r - LSE} out_r,
// parts r = 0 .. n_parts - 1 taken in order by every caller (identical results on every rank).
// Layouts: out_parts fp32 [n_parts][n_q][n_heads][512], lse_parts fp32 [n_parts][n_q][n_heads];
// a part with lse = -inf (no row) contributes nothing. One warp per (query, head): lane l owns
// dims 16 l .. 16 l + 15.
__global__ void __launch_bounds__(128) lse_merge_kernel(const float *__restrict__ out_parts,
                                                        const float *__restrict__ lse_parts, int n_parts,
                                                        int n_q, int n_heads, uint16_t *__restrict__ out,
                                                        float *__restrict__ out_f32, float *__restrict__ lse) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);   // n * n_heads + h
    if (item >= static_cast<int64_t>(n_q) * n_heads) return;
    const int64_t stride = static_cast<int64_t>(n_q) * n_heads;   // between parts
    float M = -INFINITY;
    for (int r = 0; r < n_parts; r++) M = fmaxf(M, __ldcg(lse_parts + r * stride + item));
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; e++) acc[e] = 0.0f;
    float L = 0.0f;
    for (int r = 0; r < n_parts; r++) {
        const float lr = __ldcg(lse_parts + r * stride + item);
        if (lr == -INFINITY || M == -INFINITY) continue;
        const float wr = expf(lr - M);
        L += wr;
        const float4 *src = reinterpret_cast<const float4 *>(out_parts + (r * stride + item) * kLatent) + 4 * lane;
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const float4 v = __ldcg(src + u);
            acc[4 * u] = fmaf(wr, v.x, acc[4 * u]);
            acc[4 * u + 1] = fmaf(wr, v.y, acc[4 * u + 1]);
            acc[4 * u + 2] = fmaf(wr, v.z, acc[4 * u + 2]);
            acc[4 * u + 3] = fmaf(wr, v.w, acc[4 * u + 3]);
        }
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const int64_t ob = item * kLatent + 16 * lane;
#pragma unroll
    for (int u = 0; u < 4; u++) {
        const float o0 = acc[4 * u] * inv, o1 = acc[4 * u + 1] * inv, o2 = acc[4 * u + 2] * inv, o3 = acc[4 * u + 3] * inv;
        const uint32_t lo = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o0))) |
                            (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o1))) << 16);
        const uint32_t hi = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o2))) |
                            (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o3))) << 16);
        *reinterpret_cast<uint2 *>(out + ob + 4 * u) = make_uint2(lo, hi);
        if (out_f32) *reinterpret_cast<float4 *>(out_f32 + ob + 4 * u) = make_float4(o0, o1, o2, o3);
    }
    if (lse && lane == 0) lse[item] = L > 0.0f ? M + logf(L) : -INFINITY;
}

cudaError_t launch_lse_merge(const float *out_parts, const float *lse_parts, int n_parts, int n_q, int n_heads,
                             void *out, float *out_f32, float *lse, cudaStream_t stream) {
    const int64_t items = static_cast<int64_t>(n_q) * n_heads;
    const dim3 grid(static_cast<unsigned>((items + 3) / 4));
    launch_pdl(lse_merge_kernel, grid, dim3(128), 0, stream, out_parts, lse_parts, n_parts, n_q, n_heads,
               static_cast<uint16_t *>(out), out_f32, lse);
    return cudaGetLastError();
}

}  // namespace glm
