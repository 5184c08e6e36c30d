// mla_vup.cu -- the up-projection after the absorbed (latent-space) MLA on the sm_100a tensor
// cores: each head's 512-d latent output times that head's V rows of kv_b_proj
// ("Module glm5next_dsa_ref", expand_kv: kv_b_proj maps the 512-d latent to per-head K and V;
// "GLM-5.3-Flash" pypto-lib page, 'Checkpoint shape': qk_head_dim / v_head_dim 256; 'Open
// questions an owner will hit': kv_b_proj is BF16 in the checkpoint):
//     out_v[n][h][e] = sum_d o_lat[n][h][d] * W[h (dk + dv) + dk + e][d],   e < dv, d < 512
// with W = kv_b_proj, bf16 [n_heads (dk + dv), 512] (torch Linear layout, rows grouped per head:
// the dk K rows, then the dv V rows).
//
// One CTA per (head, 128 of its dv outputs, 128 queries): D[128 queries x 128 outputs] =
// A[queries x 512] . B[outputs x 512]^T on tcgen05 (kind::f16, bf16 operands, fp32 accumulator in
// tensor memory, 32 MMAs of M = 128, N = 128, K = 16). Both operands arrive by TMA in the 128-byte
// swizzle layout: the CTA's whole 128 KB slice of W is requested first -- it is a weight, not an
// output of the preceding kernel, so under programmatic dependent launch it streams while that
// kernel still runs -- then the latent outputs, 64 dims per box, through a 4-stage ring once the
// preceding kernel has finished. Queries past n_q read as zeros (TMA bounds) and are not stored.
// For one decode query the kernel is bound by the 16.8 MB of W_v (64 heads x 256 x 512 bf16); for
// thousands of queries by the tensor cores.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace glm {

GLM_TL_TABLE(glm_tl_vup)

constexpr int kVuThreads = 128;
constexpr int kVuTile = 128;               // queries (M) and outputs (N) of a CTA
constexpr int kVuKBox = 64;                // latent dims per TMA box (128 bytes of bf16)
constexpr int kVuKBlocks = kLatent / kVuKBox;   // 8
constexpr int kVuBoxBytes = kVuTile * kVuKBox * 2;   // 16 KB
constexpr int kVuStages = 4;
constexpr uint32_t kVuWaitLimit = 1u << 22;

struct VuLayout {                          // offsets from a 1024-byte aligned base
    static constexpr int kW = 0;                                   // 8 boxes of W_v: 128 KB
    static constexpr int kA = kW + kVuKBlocks * kVuBoxBytes;       // 4 stages of o_lat: 64 KB
    static constexpr int kBar = kA + kVuStages * kVuBoxBytes;      // W full, A full[4], A empty[4], acc
    static constexpr int kTmem = kBar + 10 * 8;
    static constexpr int kBytes = kTmem + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

__global__ void __launch_bounds__(kVuThreads, 1) mla_vup_kernel(const __grid_constant__ CUtensorMap map_a,
                                                                const __grid_constant__ CUtensorMap map_w,
                                                                int n_heads, int dk, int dv, int n_q,
                                                                uint16_t *__restrict__ out_v,
                                                                float *__restrict__ out_f32) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u);
    const int tiles_e = dv / kVuTile;
    const int h = blockIdx.x / tiles_e, et = blockIdx.x % tiles_e, m0 = blockIdx.y * kVuTile;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sw = tc::smem_addr(smem + VuLayout::kW), sa = tc::smem_addr(smem + VuLayout::kA);
    const uint32_t bar0 = tc::smem_addr(smem + VuLayout::kBar);
    const uint32_t bar_w = bar0, bar_acc = bar0 + 9 * 8;
    auto bar_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_empty = [&](int s) { return bar0 + 8u * (1 + kVuStages + s); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + VuLayout::kTmem);
    GLM_TL(glm_tl_vup, 0);

    if (tid == 0) {
        tc::mbar_init(bar_w, 1);
        for (int s = 0; s < kVuStages; s++) {
            tc::mbar_init(bar_full(s), 1);
            tc::mbar_init(bar_empty(s), 1);
        }
        tc::mbar_init(bar_acc, 1);
        tc::mbar_fence_init();
        // the CTA's W_v slice first: rows h (dk + dv) + dk + 128 et .. + 127, all 512 dims
        tc::mbar_arrive_expect_tx(bar_w, kVuKBlocks * kVuBoxBytes);
        const int w_row = h * (dk + dv) + dk + et * kVuTile;
        for (int kb = 0; kb < kVuKBlocks; kb++)
            tc::tma_load_2d(sw + kb * kVuBoxBytes, &map_w, bar_w, kb * kVuKBox, w_row);
    }
    if (warp == 2) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), kVuTile);
        tc::tmem_relinquish();
        tc::fence_before_sync();
    }
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // the latent outputs are written by the preceding kernel: wait for it, then let the next start
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    GLM_TL(glm_tl_vup, 1);
    bool ok = true;
    if (warp == 0 && lane == 0) {
        // producer: 64-dim boxes of o_lat[m0 .. m0 + 127][h][.] through the ring
        asm volatile("fence.proxy.async.global;" ::: "memory");
        for (int kb = 0; kb < kVuKBlocks; kb++) {
            const int s = kb % kVuStages;
            if (kb >= kVuStages && !tc::mbar_wait(bar_empty(s), ((kb / kVuStages) - 1) & 1, kVuWaitLimit)) ok = false;
            tc::mbar_arrive_expect_tx(bar_full(s), kVuBoxBytes);
            tc::tma_load_3d(sa + s * kVuBoxBytes, &map_a, bar_full(s), kb * kVuKBox, h, m0);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        const uint32_t idesc = tc::idesc_bf16(kVuTile, kVuTile, false, false);
        if (!tc::mbar_wait(bar_w, 0, kVuWaitLimit)) ok = false;
        for (int kb = 0; kb < kVuKBlocks; kb++) {
            const int s = kb % kVuStages;
            if (!tc::mbar_wait(bar_full(s), (kb / kVuStages) & 1, kVuWaitLimit)) ok = false;
            tc::fence_after_sync();
#pragma unroll
            for (int k = 0; k < kVuKBox / 16; k++)
                tc::mma_bf16(tmem, tc::desc_sw128(sa + s * kVuBoxBytes + k * 32, 1024),
                             tc::desc_sw128(sw + kb * kVuBoxBytes + k * 32, 1024), idesc,
                             (kb > 0 || k > 0) ? 1u : 0u);
            tc::mma_commit(bar_empty(s));
        }
        tc::mma_commit(bar_acc);
    }
    __syncwarp();
    // epilogue: warp w holds queries m0 + 32 w + lane (TMEM lanes), outputs 128 et + column
    const bool done = tc::mbar_wait(bar_acc, 0, kVuWaitLimit);
    const bool all_ok = __syncthreads_and(done && ok);
    tc::fence_after_sync();
    GLM_TL(glm_tl_vup, 2);
    const int qn = m0 + warp * 32 + lane;
    const int64_t ob = (static_cast<int64_t>(qn) * n_heads + h) * dv + et * kVuTile;
#pragma unroll 1
    for (int cb = 0; cb < kVuTile; cb += 32) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + cb, r);
        tc::tmem_wait_ld();
        if (qn >= n_q) continue;
        if (!all_ok) {   // a wait gave up: NaN marks the tile invalid
#pragma unroll
            for (int e = 0; e < 32; e++) r[e] = 0x7fc00000u;
        }
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
            uint32_t p[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[e + 2 * u]), __uint_as_float(r[e + 2 * u + 1]));
                p[u] = *reinterpret_cast<const uint32_t *>(&v);
            }
            *reinterpret_cast<uint4 *>(out_v + ob + cb + e) = make_uint4(p[0], p[1], p[2], p[3]);
            if (out_f32) {
                *reinterpret_cast<float4 *>(out_f32 + ob + cb + e) =
                    make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
                *reinterpret_cast<float4 *>(out_f32 + ob + cb + e + 4) =
                    make_float4(__uint_as_float(r[e + 4]), __uint_as_float(r[e + 5]), __uint_as_float(r[e + 6]), __uint_as_float(r[e + 7]));
            }
        }
    }
    if (!all_ok) {   // wait (bounded) for this CTA's copies and MMAs still in flight before freeing
        tc::mbar_wait(bar_w, 0, kVuWaitLimit);
        tc::mbar_wait(bar_acc, 0, kVuWaitLimit);
    }
    tc::fence_before_sync();
    __syncthreads();
    GLM_TL(glm_tl_vup, 3);
    if (warp == 2) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kVuTile);
    }
}


cudaError_t launch_mla_vup(const void *o_lat, const void *w_kv_b, int n_heads, int dk, int dv, int n_q, void *out_v,
                           float *out_f32, cudaStream_t stream) {
    auto encode = tc::tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map_a, map_w;
    // o_lat bf16 [n_q][n_heads][512]: dims (512, n_heads, n_q), boxes of 64 dims x 1 head x 128 queries
    const cuuint64_t a_dim[3] = {static_cast<cuuint64_t>(kLatent), static_cast<cuuint64_t>(n_heads),
                                 static_cast<cuuint64_t>(n_q)};
    const cuuint64_t a_stride[2] = {static_cast<cuuint64_t>(kLatent) * 2,
                                    static_cast<cuuint64_t>(n_heads) * kLatent * 2};
    const cuuint32_t a_box[3] = {kVuKBox, 1, kVuTile};
    const cuuint32_t one3[3] = {1, 1, 1};
    CUresult r = encode(&map_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(o_lat), a_dim, a_stride, a_box,
                        one3, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // W bf16 [n_heads (dk + dv)][512]: boxes of 64 dims x 128 rows
    const cuuint64_t w_dim[2] = {static_cast<cuuint64_t>(kLatent), static_cast<cuuint64_t>(n_heads) * (dk + dv)};
    const cuuint64_t w_stride[1] = {static_cast<cuuint64_t>(kLatent) * 2};
    const cuuint32_t w_box[2] = {kVuKBox, kVuTile};
    const cuuint32_t one2[2] = {1, 1};
    r = encode(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(w_kv_b), w_dim, w_stride, w_box, one2,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int smem = VuLayout::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(mla_vup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(n_heads * (dv / kVuTile)), static_cast<unsigned>((n_q + kVuTile - 1) / kVuTile));
    e = launch_pdl(mla_vup_kernel, grid, dim3(kVuThreads), smem, stream, map_a, map_w, n_heads, dk, dv, n_q,
                   static_cast<uint16_t *>(out_v), out_f32);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace glm
