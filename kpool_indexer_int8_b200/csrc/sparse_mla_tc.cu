// sparse_mla_tc.cu -- sparse NoPE MLA over gathered int8 latent rows on the sm_100a tensor cores
// ("GLM-5.3 Kernels" README, 'Included': titan_mla.triton_mla_sparse_attention -- int8
// dequantisation fused in, the shared 512-d latent is both K and V, split-KV decode, fp32
// softmax and accumulation; 'The tested MLA contract': one KV head, negative index padding).
//
// One CTA per (query, chunk of 64 index entries); heads are the MMA M dimension (M = 64 for up
// to 64 heads, 128 above; missing heads are zero rows):
//   1. gather: each entry's 512 int8 codes are widened to bf16 (exact: |code| <= 127; the E4M3
//      codes of the FP8 row are exact in bf16 as well) into a shared tile C[64 rows x 512] stored as 8x8 core matrices, its fp32 scale to a register
//      file in shared memory; the query block Q[heads x 512] goes to shared memory the same way.
//   2. S = Q . C^T on tcgen05 (kind::f16, fp32 accumulator in tensor memory, 32 MMAs of K = 16).
//      C is the K-major B operand here.
//   3. softmax of the chunk, two threads per head (one TMEM lane, half of the entries each, the
//      halves' maxima and sums exchanged in shared memory): s = S * scale_j * sm_scale, m = max,
//      p = exp(s - m), l = sum p; P' = p * scale_j (the V dequantisation scale folded in) is split
//      into bf16 hi + lo so that the PV product keeps ~16 mantissa bits of P'.
//   4. O^T = C^T . P'^T: the 512 latent dims are the M dimension (4 tiles of M = 128) and the heads
//      the N dimension, so that in tensor memory one lane holds one latent dim of every head. The
//      same tile C is now the MN-major A operand (a core matrix of 8 rows x 8 dims serves both
//      products) and P' the K-major B operand; 2 terms x 4 K-steps x 4 tiles = 32 MMAs.
//   5. (m, l) and the unnormalised O of every head go to the workspace (one lane per latent dim:
//      each warp store is 32 consecutive floats of one head); the combine kernel merges the
//      chunks by log-sum-exp.
// Tensor memory: 512 columns (S in columns 0..M-1, then the 4 O^T tiles of M columns each over
// columns 0..4M-1 once S has been read).
// Every wait on the tensor cores is bounded; a timeout sets a status word and the CTA still
// frees its tensor memory and exits.
#include "common.cuh"
#include "sparse_mla.cuh"
#include "tc.cuh"

namespace glm {

constexpr int kTcRows = 64;
constexpr int kTcThreads = 256;
constexpr uint32_t kWaitLimit = 1u << 22;

template <int M>
struct TcLayout {
    static constexpr int kQ = 0;                     // M/8 head groups x 64 dim groups x 128 B
    static constexpr int kC = kQ + M * 1024;         // 8 row groups x 64 dim groups x 128 B
    static constexpr int kPhi = kC + 64 * 1024;      // M/8 head groups x 8 row groups x 128 B
    static constexpr int kPlo = kPhi + M * 128;
    static constexpr int kScl = kPlo + M * 128;      // 64 fp32 scales
    static constexpr int kRow = kScl + 256;          // 64 row indices
    static constexpr int kBar = kRow + 256;          // 2 mbarriers
    static constexpr int kTmem = kBar + 16;          // tensor-memory base address
    static constexpr int kFlag = kTmem + 16;
    static constexpr int kPmax = kFlag + 16;         // [2 column halves][128 heads] partial maxima
    static constexpr int kPl = kPmax + 2 * 128 * 4;  // [2][128] partial sums
    static constexpr int kBytes = kPl + 2 * 128 * 4;
};

__device__ __forceinline__ uint32_t codes_to_bf16x2(uint32_t w, int shift) {
    const float a = static_cast<float>(static_cast<int8_t>((w >> shift) & 0xffu));
    const float b = static_cast<float>(static_cast<int8_t>((w >> (shift + 8)) & 0xffu));
    return (__float_as_uint(a) >> 16) | (__float_as_uint(b) & 0xffff0000u);
}

// One E4M3 code (OCP E4M3FN: bias 7, subnormals) as bf16 bits -- exact: 3 mantissa bits and
// exponents 2^-9 .. 2^8 fit bf16. (Codes 0x7F / 0xFF, NaN, are never written by the store.)
__device__ __forceinline__ uint32_t e4m3_bf16_bits(uint32_t b) {
    const uint32_t s = (b & 0x80u) << 8, e = (b >> 3) & 15u, m = b & 7u;
    if (e != 0u) return s | ((e + 120u) << 7) | (m << 4);   // 2^(e-7) (1 + m/8)
    if (m == 0u) return s;
    const uint32_t p = 31u - __clz(m);                          // m 2^-9 = 2^(p-9) (1 + frac)
    return s | ((p + 118u) << 7) | (((m << (3u - p)) & 7u) << 4);
}
__device__ __forceinline__ uint32_t fp8_to_bf16x2(uint32_t w, int shift) {
    return e4m3_bf16_bits((w >> shift) & 0xffu) | (e4m3_bf16_bits((w >> (shift + 8)) & 0xffu) << 16);
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

template <int M, bool kFp8>
__global__ void __launch_bounds__(kTcThreads, 1) mla_split_tc_kernel(
    const uint16_t *__restrict__ q, int n_heads, const int8_t *__restrict__ cache, int64_t n_rows,
    const int32_t *__restrict__ rows, int width, float sm_scale, int n_chunks,
    float *__restrict__ part_acc, float *__restrict__ part_ml, int *__restrict__ status, int early_q) {
    // early_q: the query block is an input no preceding kernel writes (the one-call step), so its
    // loads are issued before waiting for the preceding kernel; only the row indices wait for it
    if (early_q) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    else pdl_begin();
    using Lay = TcLayout<M>;
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *Qs = smem + Lay::kQ;
    unsigned char *Cs = smem + Lay::kC;
    unsigned char *Phi = smem + Lay::kPhi;
    unsigned char *Plo = smem + Lay::kPlo;
    float *scl = reinterpret_cast<float *>(smem + Lay::kScl);
    int *ridx = reinterpret_cast<int *>(smem + Lay::kRow);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + Lay::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::kTmem);
    int *flag = reinterpret_cast<int *>(smem + Lay::kFlag);

    const int n = blockIdx.y, c = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ml_base = (static_cast<int64_t>(n) * n_chunks + c) * n_heads;

    // the query block (bf16 [heads x 512] as core matrices: head group stride 8192 B, dim group 128 B)
    constexpr int kQIters = M * 64 / kTcThreads;           // 16-byte query pieces per thread
    const uint16_t *qn = q + static_cast<int64_t>(n) * n_heads * kLatent;
    uint4 qv[kQIters];
#pragma unroll
    for (int it = 0; it < kQIters; it++) {
        const int i = it * kTcThreads + tid;
        const int g = i >> 5, t = i & 31;
        const int h = (g % (M / 8)) * 8 + (t & 7);
        const int dg = (g / (M / 8)) * 4 + (t >> 3);
        qv[it] = h < n_heads ? __ldg(reinterpret_cast<const uint4 *>(qn + static_cast<int64_t>(h) * kLatent) + dg)
                             : make_uint4(0u, 0u, 0u, 0u);
    }
    auto store_q = [&]() {
#pragma unroll
        for (int it = 0; it < kQIters; it++) {
            const int i = it * kTcThreads + tid;
            const int g = i >> 5, t = i & 31;
            const int hg = g % (M / 8);
            const int h = hg * 8 + (t & 7);
            const int dg = (g / (M / 8)) * 4 + (t >> 3);
            *reinterpret_cast<uint4 *>(Qs + hg * 8192 + dg * 128 + (h & 7) * 16) = qv[it];
        }
    };
    if (early_q) asm volatile("griddepcontrol.wait;" ::: "memory");   // (the query loads stay in flight)

    if (tid == 0) *flag = 0;
    __syncthreads();
    if (tid < kTcRows) {
        const int j = c * kTcRows + tid;
        const int r = j < width ? rows[static_cast<int64_t>(n) * width + j] : -1;
        const bool ok = r >= 0 && r < n_rows;
        ridx[tid] = ok ? r : -1;
        if (ok) atomicOr(flag, 1);
    }
    __syncthreads();
    if (*flag == 0) {  // no valid entry in this chunk: an empty partial
        for (int h = tid; h < n_heads; h += blockDim.x) {
            part_ml[2 * (ml_base + h)] = -INFINITY;
            part_ml[2 * (ml_base + h) + 1] = 0.0f;
        }
        return;
    }
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), 512);
        tc::tmem_relinquish();
        tc::fence_before_sync();
    }
    if (tid == 32) {
        tc::mbar_init(tc::smem_addr(&bar[0]), 1);
        tc::mbar_init(tc::smem_addr(&bar[1]), 1);
        tc::mbar_fence_init();
    }

    // 1. gather the chunk's rows (codes widened to bf16) and its scales; every global load of a
    //    thread is issued before any of them is used, so the CTA waits for one round trip
    constexpr int kRowIters = kTcRows * 32 / kTcThreads;   // 16-byte code pieces per thread
    {
        uint4 v[kRowIters];
#pragma unroll
        for (int it = 0; it < kRowIters; it++) {
            const int i = it * kTcThreads + tid;
            const int g = i >> 5, t = i & 31;
            const int j = (g & 7) * 8 + (t & 7);     // entry (row) of the chunk
            const int k = (g >> 3) * 4 + (t >> 3);   // 16-byte piece of its codes (dims 16k .. 16k+15)
            const int r = ridx[j];
            v[it] = r >= 0 ? __ldg(reinterpret_cast<const uint4 *>(cache + static_cast<int64_t>(r) * kRowBytes) + k)
                           : make_uint4(0u, 0u, 0u, 0u);
        }
        float sc = 0.0f;
        if (tid < kTcRows) {
            const int r = ridx[tid];
            if (r >= 0) sc = __ldg(reinterpret_cast<const float *>(cache + static_cast<int64_t>(r) * kRowBytes + kLatent));
        }
#pragma unroll
        for (int it = 0; it < kRowIters; it++) {
            const int i = it * kTcThreads + tid;
            const int g = i >> 5, t = i & 31;
            const int j = (g & 7) * 8 + (t & 7);
            const int k = (g >> 3) * 4 + (t >> 3);
            unsigned char *line = Cs + (j >> 3) * 8192 + (2 * k) * 128 + (j & 7) * 16;
            auto cv = [&](uint32_t w, int shift) { return kFp8 ? fp8_to_bf16x2(w, shift) : codes_to_bf16x2(w, shift); };
            *reinterpret_cast<uint4 *>(line) = make_uint4(cv(v[it].x, 0), cv(v[it].x, 16), cv(v[it].y, 0), cv(v[it].y, 16));
            *reinterpret_cast<uint4 *>(line + 128) = make_uint4(cv(v[it].z, 0), cv(v[it].z, 16), cv(v[it].w, 0), cv(v[it].w, 16));
        }
        if (tid < kTcRows) scl[tid] = sc;
        store_q();
    }
    tc::fence_proxy_async();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // 2. S = Q . C^T
    if (tid == 0) {
        const uint32_t idesc = tc::idesc_bf16(M, kTcRows, false, false);
        const uint32_t qa = tc::smem_addr(Qs), ca = tc::smem_addr(Cs);
#pragma unroll 4
        for (int ks = 0; ks < kLatent / 16; ks++)
            tc::mma_bf16(tmem, tc::desc(qa + ks * 256, 128, 8192), tc::desc(ca + ks * 256, 128, 8192), idesc,
                         ks > 0 ? 1u : 0u);
        tc::mma_commit(tc::smem_addr(&bar[0]));
    }

    // 3. softmax of the chunk on all 8 warps: warp w reads TMEM lane quadrant w % 4 (lane = head)
    //    and the columns (entries) [32 (w / 4), +32); the two halves of a head exchange their
    //    maxima and sums through shared memory
    {
        float *pmax = reinterpret_cast<float *>(smem + Lay::kPmax);
        float *pl = reinterpret_cast<float *>(smem + Lay::kPl);
        const int quad = warp & 3, hf = warp >> 2;
        if (!tc::mbar_wait(tc::smem_addr(&bar[0]), 0, kWaitLimit)) atomicOr(status, 1);
        __syncwarp();  // thread 0 arrives here after issuing the MMAs: reconverge for tcgen05.ld
        tc::fence_after_sync();
        uint32_t r[32];
        tc::tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + hf * 32, r);
        tc::tmem_wait_ld();
        const int head = (M == 128) ? quad * 32 + lane : (lane < 16 ? quad * 16 + lane : -1);
        const float k2 = sm_scale * 1.4426950408889634f;  // scores in log2 units
        float sv[32];
        float mx = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < 32; jj++) {
            const int j = hf * 32 + jj;
            sv[jj] = ridx[j] >= 0 ? __uint_as_float(r[jj]) * scl[j] * k2 : -INFINITY;
            mx = fmaxf(mx, sv[jj]);
        }
        if (head >= 0) pmax[hf * 128 + head] = mx;
        __syncthreads();
        if (head >= 0) {
            mx = fmaxf(pmax[head], pmax[128 + head]);
            float l = 0.0f;
            const bool real = head < n_heads;
#pragma unroll
            for (int rq = 0; rq < 4; rq++) {
                const int rg = hf * 4 + rq;   // row group of 8 entries
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    uint32_t hb[2], lb[2];
#pragma unroll
                    for (int u = 0; u < 2; u++) {
                        const int jj = rq * 8 + 2 * e + u, j = hf * 32 + jj;
                        const float p = ridx[j] >= 0 ? exp2f(sv[jj] - mx) : 0.0f;
                        l += p;
                        const float pp = real ? p * scl[j] : 0.0f;
                        const uint16_t h16 = bf16_rn_bits(pp);
                        hb[u] = h16;
                        lb[u] = bf16_rn_bits(pp - __uint_as_float(static_cast<uint32_t>(h16) << 16));
                    }
                    hi[e] = hb[0] | (hb[1] << 16);
                    lo[e] = lb[0] | (lb[1] << 16);
                }
                const int off = (head >> 3) * 1024 + rg * 128 + (head & 7) * 16;
                *reinterpret_cast<uint4 *>(Phi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(Plo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            pl[hf * 128 + head] = l;
            pmax[hf * 128 + head] = mx;   // (same value in both halves)
        }
        tc::fence_before_sync();
    }
    tc::fence_proxy_async();
    __syncthreads();
    if (warp < 4) {   // (m, l) of each head, natural-log units
        const float *pmax = reinterpret_cast<const float *>(smem + Lay::kPmax);
        const float *pl = reinterpret_cast<const float *>(smem + Lay::kPl);
        const int head = (M == 128) ? warp * 32 + lane : (lane < 16 ? warp * 16 + lane : -1);
        if (head >= 0 && head < n_heads) {
            part_ml[2 * (ml_base + head)] = pmax[head] * 0.6931471805599453f;
            part_ml[2 * (ml_base + head) + 1] = pl[head] + pl[128 + head];
        }
    }

    // 4. O^T = C^T . P'^T (hi and lo terms accumulate into the same columns)
    if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_bf16(128, M, true, false);
        const uint32_t ph = tc::smem_addr(Phi), pl = tc::smem_addr(Plo), ca = tc::smem_addr(Cs);
#pragma unroll
        for (int mt = 0; mt < kLatent / 128; mt++) {
#pragma unroll
            for (int ks = 0; ks < kTcRows / 16; ks++) {
                const uint64_t a = tc::desc(ca + ks * 2 * 8192 + mt * 16 * 128, 8192, 128);
                tc::mma_bf16(tmem + mt * M, a, tc::desc(ph + ks * 256, 128, 1024), idesc, ks > 0 ? 1u : 0u);
                tc::mma_bf16(tmem + mt * M, a, tc::desc(pl + ks * 256, 128, 1024), idesc, 1u);
            }
        }
        tc::mma_commit(tc::smem_addr(&bar[1]));
    }

    // 5. unnormalised O to the workspace: tile mt, lane quadrant q (latent dims 128 mt + 32 q + lane)
    {
        if (!tc::mbar_wait(tc::smem_addr(&bar[1]), 0, kWaitLimit)) atomicOr(status, 2);
        __syncwarp();
        tc::fence_after_sync();
        const int quad = warp & 3;
#pragma unroll 1
        for (int mt = warp >> 2; mt < kLatent / 128; mt += 2) {
            const int dim = mt * 128 + quad * 32 + lane;
            const uint32_t ta = tmem + (static_cast<uint32_t>(quad * 32) << 16) + mt * M;
#pragma unroll 1
            for (int hb = 0; hb < M; hb += 32) {
                uint32_t r[32];
                tc::tmem_ld32(ta + hb, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e++)
                    if (hb + e < n_heads) part_acc[(ml_base + hb + e) * kLatent + dim] = __uint_as_float(r[e]);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

int mla_tc_chunk() { return kTcRows; }

template <int M, bool kFp8>
cudaError_t launch_mla_split_tc_t(const void *q, int n_heads, const int8_t *cache, int64_t n_rows,
                                  const int32_t *rows, int n_q, int width, float sm_scale,
                                  float *part_acc, float *part_ml, int *status, cudaStream_t stream, bool early_q) {
    const int n_chunks = (width + kTcRows - 1) / kTcRows;
    const int smem = TcLayout<M>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(mla_split_tc_kernel<M, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(mla_split_tc_kernel<M, kFp8>, dim3(n_chunks, n_q), dim3(kTcThreads), smem, stream,
                   static_cast<const uint16_t *>(q), n_heads, cache, n_rows, rows, width, sm_scale, n_chunks,
                   part_acc, part_ml, status, early_q ? 1 : 0);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_mla_split_tc(const void *q, int n_heads, const int8_t *cache, int64_t n_rows,
                                const int32_t *rows, int n_q, int width, float sm_scale,
                                float *part_acc, float *part_ml, int *status, cudaStream_t stream, bool early_q,
                                bool fp8) {
    if (n_heads <= 64)
        return fp8 ? launch_mla_split_tc_t<64, true>(q, n_heads, cache, n_rows, rows, n_q, width, sm_scale, part_acc,
                                                     part_ml, status, stream, early_q)
                   : launch_mla_split_tc_t<64, false>(q, n_heads, cache, n_rows, rows, n_q, width, sm_scale, part_acc,
                                                      part_ml, status, stream, early_q);
    return fp8 ? launch_mla_split_tc_t<128, true>(q, n_heads, cache, n_rows, rows, n_q, width, sm_scale, part_acc,
                                                  part_ml, status, stream, early_q)
               : launch_mla_split_tc_t<128, false>(q, n_heads, cache, n_rows, rows, n_q, width, sm_scale, part_acc,
                                                   part_ml, status, stream, early_q);
}

}  // namespace glm
