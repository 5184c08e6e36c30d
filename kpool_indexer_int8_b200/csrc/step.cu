// step.cu -- the first kernel of a fused decode step: the store of the new latent rows ("GLM-5.3
// Kernels" README, 'Included': titan_kv.store_int8; or the FP8 or 4-bit row of "GLM on CUDA",
// --kv-dtype fp8 / fp4), the build of the new pools
// ("Module glm5next_dsa_ref", pool_states) and the zeroing of the step's cross-CTA counters, as
// three independent groups of CTAs of one launch (one warp per row, one warp per pool, 64 bytes
// per thread of zeros), so that the three short jobs overlap instead of following one another.
#include "append.cuh"
#include "kernels.cuh"

namespace glm {

GLM_TL_TABLE(glm_tl_prep)

constexpr int kPrepThreads = 256;
constexpr int kPrepWarps = kPrepThreads / 32;
constexpr int kZeroPerThread = 4;   // 16-byte stores per thread of a zeroing CTA

__global__ void __launch_bounds__(kPrepThreads) step_prep_kernel(StepPrepArgs a, int store_ctas, int pool_ctas) {
    GLM_TL(glm_tl_prep, 0);
    GLM_TL_SMID(glm_tl_prep);
    pdl_begin();
    GLM_TL(glm_tl_prep, 1);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int cta = blockIdx.x;
    if (cta < store_ctas) {
        const int64_t row = static_cast<int64_t>(cta) * kPrepWarps + warp;
        if (row < a.n_new) {
            if (a.format == kFmtFp8) store_fp8_row(a.latent, a.slots, row, reinterpret_cast<uint8_t *>(a.cache), a.n_rows);
            else if (a.format == kFmtFp4) store_fp4_row(a.latent, a.slots, row, reinterpret_cast<uint8_t *>(a.cache), a.n_rows);
            else store_int8_row(a.latent, a.slots, row, a.cache, a.n_rows);
        }
        return;
    }
    cta -= store_ctas;
    if (cta < pool_ctas) {
        const int64_t it = static_cast<int64_t>(cta) * kPrepWarps + warp;
        if (it >= static_cast<int64_t>(a.batch) * a.max_new_pools) return;
        const float4 w4 = reinterpret_cast<const float4 *>(a.ln_w)[lane];
        const float4 b4 = reinterpret_cast<const float4 *>(a.ln_b)[lane];
        const float lw[4] = {w4.x, w4.y, w4.z, w4.w}, lb[4] = {b4.x, b4.y, b4.z, b4.w};
        kpool_build_item(a.k, a.gate, a.ld_tokens, lw, lb, a.ln_eps, a.pad, a.len, a.pool_begin, a.max_new_pools,
                         a.pooled, a.ld_pools, it, a.codes, a.scales);
        return;
    }
    cta -= pool_ctas;
    const int64_t i0 = static_cast<int64_t>(cta) * kPrepThreads * kZeroPerThread + threadIdx.x;
#pragma unroll
    for (int k = 0; k < kZeroPerThread; k++) {
        const int64_t i = i0 + k * kPrepThreads;
        if (i < a.zero_n16) a.zero[i] = make_uint4(0u, 0u, 0u, 0u);
    }
}

cudaError_t launch_step_prep(const StepPrepArgs &a, cudaStream_t stream) {
    const int64_t items = static_cast<int64_t>(a.batch) * a.max_new_pools;
    const int store_ctas = static_cast<int>((a.n_new + kPrepWarps - 1) / kPrepWarps);
    const int pool_ctas = static_cast<int>((items + kPrepWarps - 1) / kPrepWarps);
    const int zero_ctas =
        static_cast<int>((a.zero_n16 + kPrepThreads * kZeroPerThread - 1) / (kPrepThreads * kZeroPerThread));
    const int total = store_ctas + pool_ctas + zero_ctas;
    if (total == 0) return cudaSuccess;
    // Keep the SMs that run these CTAs configured for the most shared memory: the fused index
    // kernel's CTAs (one per SM, ~190 KB each) start beside them under programmatic dependent
    // launch, which a smaller carve-out would hold back until these CTAs end.
    cudaError_t e = cudaFuncSetAttribute(step_prep_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    launch_pdl(step_prep_kernel, dim3(static_cast<unsigned>(total)), dim3(kPrepThreads), 0, stream, a, store_ctas,
               pool_ctas);
    return cudaGetLastError();
}

}  // namespace glm
