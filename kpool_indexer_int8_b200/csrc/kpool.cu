// kpool.cu -- k_norm LayerNorm + slot-axis softmax pooling ("Module glm5next_dsa_ref",
// pool_states and traps 1-4: LayerNorm with bias; softmax over the pool-slot axis per channel;
// pools start at the first valid token; only complete pools exist).
//
// One warp per (sequence, pool). Lane l owns channels [4l, 4l+4) of the four slot tokens: it
// loads 8 bytes of k and 8 of gate per token (each warp load is one contiguous 256-byte row),
// normalises each token with two warp reductions (mean, then biased variance), mixes the four
// slots with a per-channel softmax of the gates and stores 16 bytes of the fp32 pool row.
// HBM-bound: 4 * (256 + 256) bytes read and 512 written per pool.
#include "append.cuh"

namespace glm {

__global__ void __launch_bounds__(256) kpool_build_kernel(
    const uint16_t *__restrict__ k, const uint16_t *__restrict__ gate, int64_t ld_tokens,
    const float *__restrict__ ln_w, const float *__restrict__ ln_b, float eps,
    const int32_t *__restrict__ pad, const int32_t *__restrict__ len,
    const int32_t *__restrict__ pool_begin, int batch, int max_new_pools,
    float *__restrict__ pooled, int64_t ld_pools, int32_t *__restrict__ n_pools_out,
    int8_t *__restrict__ codes, float *__restrict__ scales) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    if (n_pools_out != nullptr && blockIdx.x == 0) {
        for (int b = threadIdx.x; b < batch; b += blockDim.x) {
            int np = len[b] > 0 ? len[b] / kKpool : 0;
            n_pools_out[b] = static_cast<int32_t>(min(static_cast<int64_t>(np), ld_pools));
        }
    }
    const float4 w4 = reinterpret_cast<const float4 *>(ln_w)[lane];
    const float4 b4 = reinterpret_cast<const float4 *>(ln_b)[lane];
    const float lw[4] = {w4.x, w4.y, w4.z, w4.w}, lb[4] = {b4.x, b4.y, b4.z, b4.w};
    const int64_t items = static_cast<int64_t>(batch) * max_new_pools;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         it < items; it += warps_total)
        kpool_build_item(k, gate, ld_tokens, lw, lb, eps, pad, len, pool_begin, max_new_pools, pooled, ld_pools, it,
                         codes, scales);
}

cudaError_t launch_kpool_build(const void *k, const void *gate, int64_t ld_tokens,
                               const float *ln_w, const float *ln_b, float eps,
                               const int32_t *pad, const int32_t *len, const int32_t *pool_begin,
                               int batch, int max_new_pools, float *pooled, int64_t ld_pools,
                               int32_t *n_pools, cudaStream_t stream, int num_sms, int8_t *codes,
                               float *scales) {
    const int warps_per_block = 8;
    int64_t items = static_cast<int64_t>(batch) * max_new_pools;
    int64_t blocks = (items + warps_per_block - 1) / warps_per_block;
    if (blocks < 1) blocks = 1;
    int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    launch_pdl(kpool_build_kernel, dim3(static_cast<unsigned>(blocks)), dim3(32 * warps_per_block), 0, stream,
               static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(gate), ld_tokens, ln_w, ln_b, eps,
               pad, len, pool_begin, batch, max_new_pools, pooled, ld_pools, n_pools, codes, scales);
    return cudaGetLastError();
}

}  // namespace glm
