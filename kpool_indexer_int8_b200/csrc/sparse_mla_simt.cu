// sparse_mla_simt.cu -- sparse NoPE MLA over gathered int8 latent rows, SIMT split-KV form
// ("GLM-5.3 Kernels" README, 'Included': titan_mla.triton_mla_sparse_attention -- int8
// dequantisation fused in, the shared 512-d latent is both K and V, split-KV decode, fp32
// softmax and accumulation; 'The tested MLA contract': one KV head, negative index padding).
//
// Split kernel: one CTA per (query, chunk of 64 index entries). The chunk's rows are copied whole
// (528 bytes, codes + scale) into shared memory with a 528-byte stride, which also keeps 16-byte
// reads of eight consecutive rows on distinct banks. Scores s = sm_scale * scale_j * (q_h . code_j)
// are fp32 dot products; the chunk's softmax state (max m, sum l) and unnormalised accumulator
// acc_h = sum_j exp(s_hj - m_h) * scale_j * code_j are written to the workspace.
// The combine kernel (shared with the tensor-core path) merges the chunks by log-sum-exp.
#include "common.cuh"
#include "sparse_mla.cuh"

namespace glm {

constexpr int kSimtChunk = 64;
constexpr int kSimtThreads = 256;
constexpr int kQStride = kLatent + 8;  // bf16 elements per q row in shared memory (16-byte pad)

__global__ void __launch_bounds__(kSimtThreads) mla_split_simt_kernel(
    const uint16_t *__restrict__ q, int n_heads, const int8_t *__restrict__ cache, int64_t n_rows,
    const int32_t *__restrict__ rows, int width, float sm_scale, int n_chunks,
    float *__restrict__ part_acc, float *__restrict__ part_ml) {
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char *crow = smem;                                               // [64][528]
    uint16_t *qs = reinterpret_cast<uint16_t *>(smem + kSimtChunk * kRowBytes);  // [Hm][520]
    float *P = reinterpret_cast<float *>(qs + n_heads * kQStride);           // [Hm][64]
    __shared__ float scl[kSimtChunk];
    __shared__ int valid[kSimtChunk];
    __shared__ int any_valid;

    const int n = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int64_t ml_base = (static_cast<int64_t>(n) * n_chunks + c) * n_heads;
    if (tid == 0) any_valid = 0;
    __syncthreads();
    if (tid < kSimtChunk) {
        const int j = c * kSimtChunk + tid;
        int r = j < width ? rows[static_cast<int64_t>(n) * width + j] : -1;
        const int ok = (r >= 0 && r < n_rows);
        valid[tid] = ok ? r : -1;
        if (ok) atomicOr(&any_valid, 1);
    }
    __syncthreads();
    if (!any_valid) {
        for (int h = tid; h < n_heads; h += blockDim.x) {
            part_ml[2 * (ml_base + h)] = -INFINITY;
            part_ml[2 * (ml_base + h) + 1] = 0.0f;
        }
        return;
    }
    // gather the rows (33 x 16 bytes each) and the queries
    for (int i = tid; i < kSimtChunk * (kRowBytes / 16); i += blockDim.x) {
        const int j = i / (kRowBytes / 16), k = i % (kRowBytes / 16);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (valid[j] >= 0) v = __ldg(reinterpret_cast<const uint4 *>(cache + static_cast<int64_t>(valid[j]) * kRowBytes) + k);
        reinterpret_cast<uint4 *>(crow + j * kRowBytes)[k] = v;
    }
    const uint16_t *qn = q + static_cast<int64_t>(n) * n_heads * kLatent;
    for (int i = tid; i < n_heads * (kLatent / 8); i += blockDim.x) {
        const int h = i / (kLatent / 8), k = i % (kLatent / 8);
        reinterpret_cast<uint4 *>(qs + h * kQStride)[k] = __ldg(reinterpret_cast<const uint4 *>(qn + h * kLatent) + k);
    }
    __syncthreads();
    if (tid < kSimtChunk) scl[tid] = *reinterpret_cast<const float *>(crow + tid * kRowBytes + kLatent);
    __syncthreads();
    // scores: thread pairs (h, j), 16-byte reads of codes, 32-byte reads of q
    for (int pr = tid; pr < n_heads * kSimtChunk; pr += blockDim.x) {
        const int h = pr / kSimtChunk, j = pr % kSimtChunk;
        float s = -INFINITY;
        if (valid[j] >= 0) {
            const uint4 *cr = reinterpret_cast<const uint4 *>(crow + j * kRowBytes);
            const uint4 *qr = reinterpret_cast<const uint4 *>(qs + h * kQStride);
            float acc = 0.0f;
#pragma unroll 4
            for (int k = 0; k < kLatent / 16; k++) {
                const uint4 cv = cr[k];
                const uint4 q0 = qr[2 * k], q1 = qr[2 * k + 1];
                const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
                const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                for (int e = 0; e < 16; e++) {
                    const float code = static_cast<float>(static_cast<int8_t>((cw[e >> 2] >> (8 * (e & 3))) & 0xffu));
                    const float qv = __uint_as_float((e & 1) ? (qw[e >> 1] & 0xffff0000u) : (qw[e >> 1] << 16));
                    acc = fmaf(qv, code, acc);
                }
            }
            s = acc * scl[j] * sm_scale;
        }
        P[h * kSimtChunk + j] = s;
    }
    __syncthreads();
    // chunk softmax per head: one warp per head, lanes over the 64 entries
    for (int h = warp; h < n_heads; h += blockDim.x >> 5) {
        float s0 = P[h * kSimtChunk + lane], s1 = P[h * kSimtChunk + lane + 32];
        const float m = warp_max(fmaxf(s0, s1));
        const float p0 = valid[lane] >= 0 ? __expf(s0 - m) : 0.0f;
        const float p1 = valid[lane + 32] >= 0 ? __expf(s1 - m) : 0.0f;
        const float l = warp_sum(p0 + p1);
        P[h * kSimtChunk + lane] = p0 * scl[lane];           // fold the V dequant scale into p
        P[h * kSimtChunk + lane + 32] = p1 * scl[lane + 32];
        if (lane == 0) {
            part_ml[2 * (ml_base + h)] = m;
            part_ml[2 * (ml_base + h) + 1] = l;
        }
    }
    __syncthreads();
    // acc[h][4d4 .. 4d4+3] = sum_j P[h][j] * code_j[...]
    for (int o = tid; o < n_heads * (kLatent / 4); o += blockDim.x) {
        const int h = o / (kLatent / 4), d4 = o % (kLatent / 4);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        const float *ph = P + h * kSimtChunk;
#pragma unroll 8
        for (int j = 0; j < kSimtChunk; j++) {
            const float pj = ph[j];
            const uint32_t cw = reinterpret_cast<const uint32_t *>(crow + j * kRowBytes)[d4];
            a0 = fmaf(pj, static_cast<float>(static_cast<int8_t>(cw & 0xffu)), a0);
            a1 = fmaf(pj, static_cast<float>(static_cast<int8_t>((cw >> 8) & 0xffu)), a1);
            a2 = fmaf(pj, static_cast<float>(static_cast<int8_t>((cw >> 16) & 0xffu)), a2);
            a3 = fmaf(pj, static_cast<float>(static_cast<int8_t>(cw >> 24)), a3);
        }
        reinterpret_cast<float4 *>(part_acc + (ml_base + h) * kLatent)[d4] = make_float4(a0, a1, a2, a3);
    }
}

size_t mla_simt_smem_bytes(int n_heads) {
    return static_cast<size_t>(kSimtChunk) * kRowBytes + static_cast<size_t>(n_heads) * kQStride * 2 +
           static_cast<size_t>(n_heads) * kSimtChunk * 4;
}

cudaError_t launch_mla_split_simt(const void *q, int n_heads, const int8_t *cache, int64_t n_rows,
                                  const int32_t *rows, int n_q, int width, float sm_scale,
                                  float *part_acc, float *part_ml, cudaStream_t stream) {
    const int n_chunks = (width + kSimtChunk - 1) / kSimtChunk;
    const size_t smem = mla_simt_smem_bytes(n_heads);
    cudaError_t e = cudaFuncSetAttribute(mla_split_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(n_chunks, n_q);
    mla_split_simt_kernel<<<grid, kSimtThreads, smem, stream>>>(
        static_cast<const uint16_t *>(q), n_heads, cache, n_rows, rows, width, sm_scale, n_chunks,
        part_acc, part_ml);
    return cudaGetLastError();
}

int mla_simt_chunk() { return kSimtChunk; }

}  // namespace glm
