// mla_combine.cu -- log-sum-exp merge of split-KV partial softmax states (the final combine of
// the split-KV decode named in "GLM-5.3 Kernels" README, 'Included': titan_mla ... split-KV).
//
//   M = max_c m_c,  L = sum_c l_c e^{m_c - M},  out = (sum_c e^{m_c - M} acc_c) / L,
//   lse = M + log L.
// Chunks with l = 0 (no valid entry) are skipped without reading their accumulator.
// One CTA of 128 threads per (query, head); thread t owns output columns [4t, 4t + 4).
#include "common.cuh"
#include "sparse_mla.cuh"

namespace glm {

constexpr int kMaxCombineChunks = 1024;  // 65536 / 64

__global__ void __launch_bounds__(128) mla_combine_kernel(const float *__restrict__ part_acc,
                                                          const float *__restrict__ part_ml,
                                                          int n_heads, int n_chunks,
                                                          uint16_t *__restrict__ out,
                                                          float *__restrict__ out_f32,
                                                          float *__restrict__ lse) {
    pdl_begin();
    __shared__ float wgt[kMaxCombineChunks];
    __shared__ float red[4];
    const int h = blockIdx.x, n = blockIdx.y, t = threadIdx.x;
    const int64_t base = static_cast<int64_t>(n) * n_chunks * n_heads + h;
    // every chunk's (m, l) at once: one round trip instead of one per chunk
    float mx = -INFINITY;
    for (int c = t; c < n_chunks; c += blockDim.x) {
        const float2 ml = *reinterpret_cast<const float2 *>(part_ml + 2 * (base + static_cast<int64_t>(c) * n_heads));
        wgt[c] = ml.y > 0.0f ? ml.x : -INFINITY;   // the chunk's max, or -inf if it had no entry
        if (ml.y > 0.0f) mx = fmaxf(mx, ml.x);
    }
    mx = warp_max(mx);
    if ((t & 31) == 0) red[t >> 5] = mx;
    __syncthreads();
    const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    float Lp = 0.0f;
    for (int c = t; c < n_chunks; c += blockDim.x) {
        const float m = wgt[c];
        const float wc = (m == -INFINITY || M == -INFINITY) ? 0.0f : expf(m - M);
        wgt[c] = wc;
        Lp = fmaf(part_ml[2 * (base + static_cast<int64_t>(c) * n_heads) + 1], wc, Lp);
    }
    Lp = warp_sum(Lp);
    if ((t & 31) == 0) red[t >> 5] = Lp;
    __syncthreads();
    const float L = (red[0] + red[1]) + (red[2] + red[3]);
    // weighted sum of the chunk accumulators, four chunks in flight per thread
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    int c = 0;
    for (; c + 4 <= n_chunks; c += 4) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; u++)
            v[u] = wgt[c + u] > 0.0f ? reinterpret_cast<const float4 *>(part_acc + (base + static_cast<int64_t>(c + u) * n_heads) * kLatent)[t]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const float wc = wgt[c + u];
            a.x = fmaf(wc, v[u].x, a.x);
            a.y = fmaf(wc, v[u].y, a.y);
            a.z = fmaf(wc, v[u].z, a.z);
            a.w = fmaf(wc, v[u].w, a.w);
        }
    }
    for (; c < n_chunks; c++) {
        const float wc = wgt[c];
        if (!(wc > 0.0f)) continue;
        const float4 v = reinterpret_cast<const float4 *>(part_acc + (base + static_cast<int64_t>(c) * n_heads) * kLatent)[t];
        a.x = fmaf(wc, v.x, a.x);
        a.y = fmaf(wc, v.y, a.y);
        a.z = fmaf(wc, v.z, a.z);
        a.w = fmaf(wc, v.w, a.w);
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const float o[4] = {a.x * inv, a.y * inv, a.z * inv, a.w * inv};
    const int64_t ob = (static_cast<int64_t>(n) * n_heads + h) * kLatent + 4 * t;
    uint32_t lo = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[0]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[1]))) << 16);
    uint32_t hi = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[2]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[3]))) << 16);
    *reinterpret_cast<uint2 *>(out + ob) = make_uint2(lo, hi);
    if (out_f32) *reinterpret_cast<float4 *>(out_f32 + ob) = make_float4(o[0], o[1], o[2], o[3]);
    if (lse && t == 0) lse[static_cast<int64_t>(n) * n_heads + h] = L > 0.0f ? M + logf(L) : -INFINITY;
}

cudaError_t launch_mla_combine(const float *part_acc, const float *part_ml, int n_q, int n_heads,
                               int n_chunks, void *out, float *out_f32, float *lse,
                               cudaStream_t stream) {
    dim3 grid(n_heads, n_q);
    launch_pdl(mla_combine_kernel, dim3(grid), dim3(128), 0, stream, part_acc, part_ml, n_heads, n_chunks,
                                                 static_cast<uint16_t *>(out), out_f32, lse);
    return cudaGetLastError();
}

}  // namespace glm
