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

constexpr int kMaxCombineChunks = 1024;  // 65536 / 64
constexpr int kCombineThreads = 512;
constexpr int kChunkGroups = kCombineThreads / (kLatent / 4);   // 4 groups of 128 threads
constexpr int kFirstLoads = 9;   // chunks per thread whose accumulators load with the (m, l) pairs

__device__ __forceinline__ void fma4(float4 &a, float w, const float4 &v) {
    a.x = fmaf(w, v.x, a.x);
    a.y = fmaf(w, v.y, a.y);
    a.z = fmaf(w, v.z, a.z);
    a.w = fmaf(w, v.w, a.w);
}

// One CTA of 512 threads per (head, query): thread t owns output columns [4 (t % 128), +4) of
// chunk group t / 128 (chunks c = group, group + 4, ...). The accumulators of its first
// kFirstLoads chunks are loaded together with every chunk's (m, l), so that one round trip to L2
// serves both; the weights follow from the (m, l) pairs, the rest of the chunks (if any) load 8 at
// a time, and the 4 group sums are added in shared memory. A chunk without a valid entry (l = 0)
// was never written: its accumulator is dropped, never multiplied.
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
    if (poison && __ldcg(poison) != 0) {   // a split CTA gave up a wait: its partial is missing
        const int64_t ob = (static_cast<int64_t>(blockIdx.y) * n_heads + blockIdx.x) * kLatent;
        for (int i = threadIdx.x; i < kLatent; i += blockDim.x) {
            out[ob + i] = 0x7fc0u;   // bf16 NaN
            if (out_f32) out_f32[ob + i] = __int_as_float(0x7fc00000);
        }
        if (lse && threadIdx.x == 0) lse[static_cast<int64_t>(blockIdx.y) * n_heads + blockIdx.x] = __int_as_float(0x7fc00000);
        return;
    }
    __shared__ float wgt[kMaxCombineChunks];
    __shared__ float lsum[kMaxCombineChunks];
    __shared__ float red[kCombineThreads / 32];
    __shared__ float4 part[kChunkGroups - 1][kLatent / 4];
    const int h = blockIdx.x, n = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t base = static_cast<int64_t>(n) * n_chunks * n_heads + h;
    const int col = t % (kLatent / 4), grp = t / (kLatent / 4);
    auto acc_at = [&](int c) {
        return __ldcg(reinterpret_cast<const float4 *>(part_acc + (base + static_cast<int64_t>(c) * n_heads) * kLatent) + col);
    };
    float4 v[kFirstLoads];
#pragma unroll
    for (int u = 0; u < kFirstLoads; u++) {
        const int cu = grp + u * kChunkGroups;
        v[u] = cu < n_chunks ? acc_at(cu) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // every chunk's (m, l); M = the largest m of a chunk with an entry
    float mx = -INFINITY;
    for (int c = t; c < n_chunks; c += kCombineThreads) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(part_ml + 2 * (base + static_cast<int64_t>(c) * n_heads)));
        wgt[c] = ml.y > 0.0f ? ml.x : -INFINITY;
        lsum[c] = ml.y;
        if (ml.y > 0.0f) mx = fmaxf(mx, ml.x);
    }
    mx = warp_max(mx);
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float M = lane < kCombineThreads / 32 ? red[lane] : -INFINITY;
    M = warp_max(M);
    __syncthreads();
    float Lp = 0.0f;
    for (int c = t; c < n_chunks; c += kCombineThreads) {
        const float m = wgt[c];
        const float wc = (m == -INFINITY || M == -INFINITY) ? 0.0f : expf(m - M);
        wgt[c] = wc;
        Lp = fmaf(lsum[c], wc, Lp);
    }
    Lp = warp_sum(Lp);
    if (lane == 0) red[warp] = Lp;
    __syncthreads();
    float L = lane < kCombineThreads / 32 ? red[lane] : 0.0f;
    L = warp_sum(L);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kFirstLoads; u++) {
        const int cu = grp + u * kChunkGroups;
        if (cu < n_chunks && wgt[cu] > 0.0f) fma4(a, wgt[cu], v[u]);
    }
    int c = grp + kFirstLoads * kChunkGroups;
    for (; c + 7 * kChunkGroups < n_chunks; c += 8 * kChunkGroups) {
        float4 r[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int cu = c + u * kChunkGroups;
            r[u] = wgt[cu] > 0.0f ? acc_at(cu) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const float wc = wgt[c + u * kChunkGroups];
            if (wc > 0.0f) fma4(a, wc, r[u]);
        }
    }
    for (; c < n_chunks; c += kChunkGroups) {
        const float wc = wgt[c];
        if (wc > 0.0f) fma4(a, wc, acc_at(c));
    }
    if (grp > 0) part[grp - 1][col] = a;
    __syncthreads();
    if (grp > 0) return;
#pragma unroll
    for (int g2 = 0; g2 < kChunkGroups - 1; g2++) {
        const float4 b = part[g2][col];
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const float o[4] = {a.x * inv, a.y * inv, a.z * inv, a.w * inv};
    const int64_t ob = (static_cast<int64_t>(n) * n_heads + h) * kLatent + 4 * col;
    uint32_t lo = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[0]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[1]))) << 16);
    uint32_t hi = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[2]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[3]))) << 16);
    *reinterpret_cast<uint2 *>(out + ob) = make_uint2(lo, hi);
    if (out_f32) *reinterpret_cast<float4 *>(out_f32 + ob) = make_float4(o[0], o[1], o[2], o[3]);
    GLM_TL(glm_tl_combine, 2);
    if (lse && t == 0) lse[static_cast<int64_t>(n) * n_heads + h] = L > 0.0f ? M + logf(L) : -INFINITY;
}

cudaError_t launch_mla_combine(const float *part_acc, const float *part_ml, int n_q, int n_heads,
                               int n_chunks, void *out, float *out_f32, float *lse,
                               cudaStream_t stream, const int *poison) {
    dim3 grid(n_heads, n_q);
    launch_pdl(mla_combine_kernel, dim3(grid), dim3(kCombineThreads), 0, stream, part_acc, part_ml, n_heads,
               n_chunks, static_cast<uint16_t *>(out), out_f32, lse, poison);
    return cudaGetLastError();
}

}  // namespace glm
