// store_int8.cu -- BF16 latent -> 528-byte int8 cache row ("GLM-5.3 Kernels" README, 'Included':
// titan_kv.store_int8: 512 int8 values, one fp32 scale, 12 zero padding bytes, scattered by slot).
//
// One warp per latent row. Lane l owns elements [16l, 16l+16): two 16-byte loads of bf16, a warp
// max for amax, an IEEE fp32 quotient per element rounded half-to-even, then one 16-byte store of
// its 16 codes. Lane 0 also stores the scale and the 12 zero bytes as a final 16-byte chunk.
// The row stride of 528 = 33 * 16 bytes keeps every store 16-byte aligned.
// HBM-bound: 1024 bytes read + 528 written + 8 bytes of slot per row.
#include "common.cuh"

namespace glm {

__global__ void __launch_bounds__(256) store_int8_kernel(const uint16_t *__restrict__ latent,
                                                         const int64_t *__restrict__ slots,
                                                         int64_t n, int8_t *__restrict__ cache,
                                                         int64_t n_rows) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         row < n; row += warps_total) {
        const int64_t slot = slots[row];
        if (slot < 0 || slot >= n_rows) continue;  // padding (or outside the contract): no write
        const uint4 *src = reinterpret_cast<const uint4 *>(latent + row * kLatent) + lane * 2;
        uint4 v0 = __ldcs(src), v1 = __ldcs(src + 1);
        uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float x[16];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            amax = fmaxf(amax, fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1])));
        }
        amax = warp_max(amax);
        amax = fmaxf(amax, 1e-4f);
        const float scale = __fdiv_rn(amax, 127.0f);
        uint32_t packed[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            uint32_t p = 0;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                int c = __float2int_rn(__fdiv_rn(x[4 * i + j], scale));
                c = max(-127, min(127, c));
                p |= (static_cast<uint32_t>(c) & 0xffu) << (8 * j);
            }
            packed[i] = p;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(cache + slot * kRowBytes);
        dst[lane] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        if (lane == 0) dst[32] = make_uint4(__float_as_uint(scale), 0u, 0u, 0u);
    }
}

cudaError_t launch_store_int8(const void *latent, const int64_t *slots, int64_t n, int8_t *cache,
                              int64_t n_rows, cudaStream_t stream, int num_sms) {
    if (n == 0) return cudaSuccess;
    const int warps_per_block = 8;
    int64_t blocks = (n + warps_per_block - 1) / warps_per_block;
    int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    launch_pdl(store_int8_kernel, dim3(static_cast<unsigned>(blocks)), dim3(32 * warps_per_block), 0, stream,
               static_cast<const uint16_t *>(latent), slots, n, cache, n_rows);
    return cudaGetLastError();
}

}  // namespace glm
