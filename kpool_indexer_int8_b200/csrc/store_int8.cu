// store_int8.cu -- BF16 latent -> 528-byte int8 cache row ("GLM-5.3 Kernels" README, 'Included':
// titan_kv.store_int8: 512 int8 values, one fp32 scale, 12 zero padding bytes, scattered by slot).
//
// One warp per latent row. Lane l owns elements [16l, 16l+16): two 16-byte loads of bf16, a warp
// max for amax, an IEEE fp32 quotient per element rounded half-to-even, then one 16-byte store of
// its 16 codes. Lane 0 also stores the scale and the 12 zero bytes as a final 16-byte chunk.
// The row stride of 528 = 33 * 16 bytes keeps every store 16-byte aligned.
// HBM-bound: 1024 bytes read + 528 written + 8 bytes of slot per row.
// store_fp8_kernel writes the FP8 twin of the row (E4M3 codes, scale = amax / 448) the same way,
// store_fp4_kernel the 304-byte 4-bit row (E2M1 codes, E4M3 block scales, an fp32 row scale).
#include "append.cuh"

namespace glm {

__global__ void __launch_bounds__(256) store_int8_kernel(const uint16_t *__restrict__ latent,
                                                         const int64_t *__restrict__ slots,
                                                         int64_t n, int8_t *__restrict__ cache,
                                                         int64_t n_rows) {
    pdl_begin();
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         row < n; row += warps_total)
        store_int8_row(latent, slots, row, cache, n_rows);
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

__global__ void __launch_bounds__(256) store_fp8_kernel(const uint16_t *__restrict__ latent,
                                                        const int64_t *__restrict__ slots,
                                                        int64_t n, uint8_t *__restrict__ cache,
                                                        int64_t n_rows) {
    pdl_begin();
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         row < n; row += warps_total)
        store_fp8_row(latent, slots, row, cache, n_rows);
}

cudaError_t launch_store_fp8(const void *latent, const int64_t *slots, int64_t n, uint8_t *cache,
                             int64_t n_rows, cudaStream_t stream, int num_sms) {
    if (n == 0) return cudaSuccess;
    const int warps_per_block = 8;
    int64_t blocks = (n + warps_per_block - 1) / warps_per_block;
    int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    launch_pdl(store_fp8_kernel, dim3(static_cast<unsigned>(blocks)), dim3(32 * warps_per_block), 0, stream,
               static_cast<const uint16_t *>(latent), slots, n, cache, n_rows);
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256) store_fp4_kernel(const uint16_t *__restrict__ latent,
                                                        const int64_t *__restrict__ slots,
                                                        int64_t n, uint8_t *__restrict__ cache,
                                                        int64_t n_rows) {
    pdl_begin();
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         row < n; row += warps_total)
        store_fp4_row(latent, slots, row, cache, n_rows);
}

cudaError_t launch_store_fp4(const void *latent, const int64_t *slots, int64_t n, uint8_t *cache,
                             int64_t n_rows, cudaStream_t stream, int num_sms) {
    if (n == 0) return cudaSuccess;
    const int warps_per_block = 8;
    int64_t blocks = (n + warps_per_block - 1) / warps_per_block;
    int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    launch_pdl(store_fp4_kernel, dim3(static_cast<unsigned>(blocks)), dim3(32 * warps_per_block), 0, stream,
               static_cast<const uint16_t *>(latent), slots, n, cache, n_rows);
    return cudaGetLastError();
}

}  // namespace glm
