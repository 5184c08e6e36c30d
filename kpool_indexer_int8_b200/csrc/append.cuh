// append.cuh -- per-warp bodies of the two per-step appends: the int8 store of one new latent
// row ("GLM-5.3 Kernels" README, 'Included': titan_kv.store_int8) and the build of one new pool
// ("Module glm5next_dsa_ref", pool_states: k_norm LayerNorm with bias, softmax over the pool-slot
// axis per channel). Used by their own kernels and by the fused decode step's first kernel.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace glm {

// Row `row` of the batch (one warp; every lane calls).
__device__ __forceinline__ void store_int8_row(const uint16_t *__restrict__ latent, const int64_t *__restrict__ slots,
                                               int64_t row, int8_t *__restrict__ cache, int64_t n_rows) {
    const int lane = threadIdx.x & 31;
    const int64_t slot = slots[row];
    if (slot < 0 || slot >= n_rows) return;  // padding (or outside the contract): no write
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

// The E4M3 code of x (nearest value, ties to the even code, saturating at +-448; the hardware
// conversion, given x twice so that the code's byte position is not in question).
__device__ __forceinline__ uint32_t e4m3_code(float x) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(x), "f"(x));
    return static_cast<uint32_t>(d) & 0xffu;
}

// Eight E2M1 codes (nearest value, ties to the even code, saturating at +-6, the sign kept; the
// hardware conversion) packed low nibble first: v[0] in bits 0-3, v[1] in bits 4-7, ... (each
// conversion puts its first operand in the high nibble of its byte).
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// The FP8 twin of store_int8_row (the FP8 latent cache of "GLM on CUDA", --kv-dtype fp8): the same
// 528-byte row with E4M3 codes and scale = max(amax, 1e-4) / 448. One warp; every lane calls.
__device__ __forceinline__ void store_fp8_row(const uint16_t *__restrict__ latent, const int64_t *__restrict__ slots,
                                              int64_t row, uint8_t *__restrict__ cache, int64_t n_rows) {
    const int lane = threadIdx.x & 31;
    const int64_t slot = slots[row];
    if (slot < 0 || slot >= n_rows) return;  // padding (or outside the contract): no write
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
    const float scale = __fdiv_rn(amax, 448.0f);
    uint32_t packed[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        uint32_t p = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) p |= e4m3_code(__fdiv_rn(x[4 * i + j], scale)) << (8 * j);
        packed[i] = p;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(cache + slot * kRowBytes);
    dst[lane] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    if (lane == 0) dst[32] = make_uint4(__float_as_uint(scale), 0u, 0u, 0u);
}

// The 4-bit row (the 4-bit latent cache of "GLM on CUDA", --kv-dtype fp4): E2M1 codes with one
// E4M3 scale per 16 values and one fp32 scale per row, 304 bytes:
//   s_row = max(amax, 1e-4) / 2688, e_k = E4M3(bmax_k / (6 s_row)), d_k = value(e_k) s_row,
//   code = E2M1(x / d_k) (0 where d_k = 0), each step one IEEE fp32 operation; both conversions
//   are the hardware's (nearest, ties to even, saturating). Lane l holds block l (dims 16 l ..).
__device__ __forceinline__ void store_fp4_row(const uint16_t *__restrict__ latent, const int64_t *__restrict__ slots,
                                              int64_t row, uint8_t *__restrict__ cache, int64_t n_rows) {
    const int lane = threadIdx.x & 31;
    const int64_t slot = slots[row];
    if (slot < 0 || slot >= n_rows) return;  // padding (or outside the contract): no write
    const uint4 *src = reinterpret_cast<const uint4 *>(latent + row * kLatent) + lane * 2;
    uint4 v0 = __ldcs(src), v1 = __ldcs(src + 1);
    uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float x[16];
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        bmax = fmaxf(bmax, fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1])));
    }
    const float amax = fmaxf(warp_max(bmax), 1e-4f);
    const float s_row = __fdiv_rn(amax, 2688.0f);
    const uint32_t e = e4m3_code(__fdiv_rn(bmax, __fmul_rn(6.0f, s_row)));
    const __half_raw ev = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(e), __NV_E4M3);
    const float d = __fmul_rn(__half2float(__half(ev)), s_row);
    uint32_t packed[2];
#pragma unroll
    for (int i = 0; i < 2; i++) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; j++) v[j] = d > 0.0f ? __fdiv_rn(x[8 * i + j], d) : 0.0f;
        packed[i] = e2m1x8(v);
    }
    uint8_t *dst = cache + slot * kFp4RowBytes;
    reinterpret_cast<uint2 *>(dst)[lane] = make_uint2(packed[0], packed[1]);
    dst[kFp4ScalesAt + lane] = static_cast<uint8_t>(e);
    if (lane == 0) *reinterpret_cast<uint4 *>(dst + kFp4RowScaleAt) = make_uint4(__float_as_uint(s_row), 0u, 0u, 0u);
}

// Item `it` = (sequence b, i-th new pool) of a build (one warp; every lane calls). lw / lb: this
// lane's four LayerNorm weights and biases.
__device__ __forceinline__ void kpool_build_item(const uint16_t *__restrict__ k, const uint16_t *__restrict__ gate,
                                                 int64_t ld_tokens, const float (&lw)[4], const float (&lb)[4],
                                                 float eps, const int32_t *__restrict__ pad,
                                                 const int32_t *__restrict__ len,
                                                 const int32_t *__restrict__ pool_begin, int max_new_pools,
                                                 float *__restrict__ pooled, int64_t ld_pools, int64_t it,
                                                 int8_t *__restrict__ codes = nullptr,
                                                 float *__restrict__ scales = nullptr) {
    const int lane = threadIdx.x & 31;
    const int b = static_cast<int>(it / max_new_pools);
    const int i = static_cast<int>(it % max_new_pools);
    const int p = (pool_begin ? pool_begin[b] : 0) + i;
    const int n_seq_pools = len[b] > 0 ? len[b] / kKpool : 0;
    if (p < 0 || p >= n_seq_pools || p >= ld_pools) return;
    const int64_t t0 = static_cast<int64_t>(b) * ld_tokens + pad[b] + static_cast<int64_t>(p) * kKpool;
    float y[kKpool][4], g[kKpool][4];
#pragma unroll
    for (int s = 0; s < kKpool; s++) {
        const uint2 kv = reinterpret_cast<const uint2 *>(k + (t0 + s) * kIdxDim)[lane];
        const uint2 gv = reinterpret_cast<const uint2 *>(gate + (t0 + s) * kIdxDim)[lane];
        float x[4] = {__uint_as_float(kv.x << 16), __uint_as_float(kv.x & 0xffff0000u),
                      __uint_as_float(kv.y << 16), __uint_as_float(kv.y & 0xffff0000u)};
        g[s][0] = __uint_as_float(gv.x << 16);
        g[s][1] = __uint_as_float(gv.x & 0xffff0000u);
        g[s][2] = __uint_as_float(gv.y << 16);
        g[s][3] = __uint_as_float(gv.y & 0xffff0000u);
        const float mean = warp_sum((x[0] + x[1]) + (x[2] + x[3])) * (1.0f / kIdxDim);
        float d0 = x[0] - mean, d1 = x[1] - mean, d2 = x[2] - mean, d3 = x[3] - mean;
        const float var = warp_sum((d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3)) * (1.0f / kIdxDim);
        const float inv = 1.0f / sqrtf(var + eps);
        y[s][0] = d0 * inv * lw[0] + lb[0];
        y[s][1] = d1 * inv * lw[1] + lb[1];
        y[s][2] = d2 * inv * lw[2] + lb[2];
        y[s][3] = d3 * inv * lw[3] + lb[3];
    }
    float out[4];
#pragma unroll
    for (int c = 0; c < 4; c++) {
        float m = fmaxf(fmaxf(g[0][c], g[1][c]), fmaxf(g[2][c], g[3][c]));
        float num = 0.0f, den = 0.0f;
#pragma unroll
        for (int s = 0; s < kKpool; s++) {
            float e = expf(g[s][c] - m);
            den += e;
            num += e * y[s][c];
        }
        out[c] = num / den;
    }
    const int64_t row = static_cast<int64_t>(b) * ld_pools + p;
    if (codes == nullptr) {
        reinterpret_cast<float4 *>(pooled + row * kIdxDim)[lane] = make_float4(out[0], out[1], out[2], out[3]);
        return;
    }
    // INT8 indexer state: the row's amax (floored at 1e-4) over 127 is the scale; codes are the
    // IEEE fp32 quotients rounded half to even, clamped to +-127 (the latent cache rows' recipe)
    float amax = fmaxf(fmaxf(fabsf(out[0]), fabsf(out[1])), fmaxf(fabsf(out[2]), fabsf(out[3])));
    amax = fmaxf(warp_max(amax), 1e-4f);
    const float scale = __fdiv_rn(amax, 127.0f);
    uint32_t packed = 0;
#pragma unroll
    for (int c = 0; c < 4; c++) {
        int q = __float2int_rn(__fdiv_rn(out[c], scale));
        q = max(-127, min(127, q));
        packed |= (static_cast<uint32_t>(q) & 0xffu) << (8 * c);
    }
    reinterpret_cast<uint32_t *>(codes + row * kIdxDim)[lane] = packed;
    if (lane == 0) scales[row] = scale;
}

}  // namespace glm
