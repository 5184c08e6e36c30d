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

__global__ void __launch_bounds__(128) mla_combine_kernel(const float *__restrict__ part_acc,
                                                          const float *__restrict__ part_ml,
                                                          int n_heads, int n_chunks,
                                                          uint16_t *__restrict__ out,
                                                          float *__restrict__ out_f32,
                                                          float *__restrict__ lse) {
    const int h = blockIdx.x, n = blockIdx.y, t = threadIdx.x;
    const int64_t base = static_cast<int64_t>(n) * n_chunks * n_heads + h;
    float M = -INFINITY;
    for (int c = 0; c < n_chunks; c++) {
        const float l = part_ml[2 * (base + static_cast<int64_t>(c) * n_heads) + 1];
        if (l > 0.0f) M = fmaxf(M, part_ml[2 * (base + static_cast<int64_t>(c) * n_heads)]);
    }
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.0f;
    if (M != -INFINITY) {
        for (int c = 0; c < n_chunks; c++) {
            const int64_t idx = base + static_cast<int64_t>(c) * n_heads;
            const float l = part_ml[2 * idx + 1];
            if (!(l > 0.0f)) continue;
            const float wgt = expf(part_ml[2 * idx] - M);
            L = fmaf(l, wgt, L);
            const float4 v = reinterpret_cast<const float4 *>(part_acc + idx * kLatent)[t];
            a.x = fmaf(wgt, v.x, a.x);
            a.y = fmaf(wgt, v.y, a.y);
            a.z = fmaf(wgt, v.z, a.z);
            a.w = fmaf(wgt, v.w, a.w);
        }
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
    mla_combine_kernel<<<grid, 128, 0, stream>>>(part_acc, part_ml, n_heads, n_chunks,
                                                 static_cast<uint16_t *>(out), out_f32, lse);
    return cudaGetLastError();
}

}  // namespace glm
