// sparse_mla_tc.cu -- sparse NoPE MLA over gathered int8 latent rows on the sm_100a tensor cores
// ("GLM-5.3 Kernels" README, 'Included': titan_mla.triton_mla_sparse_attention -- int8
// dequantisation fused in, the shared 512-d latent is both K and V, split-KV decode, fp32
// softmax and accumulation; 'The tested MLA contract': one KV head, negative index padding).
//
// One CTA per (query, chunk of ROWS index entries, group of NH heads); the rows of a chunk are
// the MMA M dimension, the heads the N dimension:
//   1. the query block of the head group goes to shared memory as fp16, each head scaled by the
//      power of two 2^e_h that puts its largest magnitude in [2^14, 2^15) (every bf16 value of
//      magnitude >= 2^-17 after scaling is exact in fp16; the scores are multiplied back by
//      2^-e_h); in the one-call step its loads are issued before the kernel waits for the index
//      lists;
//   2. gather: every thread requests its 16-byte pieces of the chunk's rows at once (all of a
//      chunk's loads in flight together: one round trip), and the row scales; while they are in
//      flight the query block is staged; the codes are then widened in registers to fp16 (exact:
//      |code| <= 127; E4M3 codes are exact in fp16 as well; a 4-bit row's E2M1 code times its
//      E4M3 block scale too) and stored as a tile C[ROWS x 512] of 8x8 core matrices -- the int8
//      codes through byte permutes and one packed subtraction (1024 + code + 128 built as fp16
//      bits, minus 1152), no integer conversions;
//   3. S^T = C . Q^T on tcgen05 (kind::f16, fp32 accumulator in tensor memory: lane = row,
//      column = head), 32 MMAs of K = 16;
//   4. softmax over the chunk's rows for each head: one thread per row and half of the heads;
//      per-head maxima and sums by a transposing warp butterfly (V - 1 + log shuffles for V
//      values) and four quadrant partials in shared memory; p = exp2(s - m) with
//      s = S * scale_row * sm_scale * log2(e) * 2^-e_h; P' = p * scale_row / scale_max (the
//      chunk's largest row scale, so P' <= 1) as an fp16 hi + lo pair;
//   5. O^T = C^T . [P'_hi | P'_lo]^T: the 512 latent dims are M (4 tiles of 128), the hi and lo
//      heads side by side are N = 2 NH, K = ROWS; the tile C is now the MN-major A operand (one
//      core matrix of 8 rows x 8 dims serves both products);
//   6. acc = scale_max * (O_hi + O_lo) and (m, l) of each head go to the workspace (lane = latent
//      dim: every warp store is 32 consecutive floats of one head); the combine kernel merges the
//      chunks by log-sum-exp.
// Every wait on the tensor cores is bounded; a timeout sets a status bit, waits (bounded) for this
// CTA's MMAs still in flight, frees the tensor memory and leaves the partial unwritten.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "sparse_mla.cuh"
#include "tc.cuh"

namespace glm {

GLM_TL_TABLE(glm_tl_split)

constexpr int kMlaThreads = 256;
constexpr uint32_t kMlaWaitLimit = 1u << 22;

template <int ROWS, int NH>
struct MlaLayout {
    static constexpr int kPBytes = ROWS * 4 * NH;                     // ROWS x 2 NH fp16 (hi | lo)
    static constexpr int kC = 0;                                      // ROWS/8 row groups x 64 dim groups x 128 B
    static constexpr int kP = kC + ROWS * 1024;                       // P', core matrices of 8 rows x 8 heads
    static constexpr int kQ = kP + kPBytes;                           // NH/8 x 64 x 128 B
    static constexpr int kScl = kQ + NH * 1024;                       // ROWS fp32 row scales
    static constexpr int kRow = kScl + ROWS * 4;                      // ROWS row indices
    static constexpr int kRed = kRow + ROWS * 4;                      // [4 quadrants][NH] partial maxima
    static constexpr int kRed2 = kRed + 4 * NH * 4;                   // [4][NH] partial sums
    static constexpr int kQk = kRed2 + 4 * NH * 4;                    // NH fp32 score factors
    static constexpr int kQmax = kQk + NH * 4;                        // NH uint32 |q| maxima (bf16 bits)
    static constexpr int kWords = kQmax + NH * 4;                     // [0] scale max bits, [1] tmem base
    static constexpr int kBar = kWords + 16;                          // 2 mbarriers
    static constexpr int kBytes = kBar + 2 * 8;
    static_assert(kQ % 16 == 0 && kP % 16 == 0 && kBar % 8 == 0, "alignment");
};

// Four int8 codes (one little-endian word) as four exact fp16 values (two fp16x2 words).
__device__ __forceinline__ void codes_to_f16x4(uint32_t w, uint32_t &lo, uint32_t &hi) {
    const uint32_t t = w ^ 0x80808080u;                          // each code c as the byte c + 128
    const uint32_t a = __byte_perm(t, 0x64646464u, 0x5140u);     // fp16 bits 0x64bb = 1024 + c + 128
    const uint32_t b = __byte_perm(t, 0x64646464u, 0x5342u);
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(0x64806480u));   // - 1152 (exact)
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(0x64806480u));
}
// Eight E2M1 codes (one word, low nibble first) as eight fp16 values times the fp16 block scale
// sc2 (in both halves): exact, since a 2-bit by 4-bit significand product of magnitude in
// [2^-10, 2688] is an fp16 normal.
__device__ __forceinline__ void fp4_to_f16x8(uint32_t w, uint32_t sc2, uint32_t (&o)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]) : "r"(w));
#pragma unroll
    for (int i = 0; i < 4; i++) asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(o[i]) : "r"(sc2));
}
// Four E4M3 codes as four exact fp16 values (hardware conversion of code pairs).
__device__ __forceinline__ void fp8_to_f16x4(uint32_t w, uint32_t &lo, uint32_t &hi) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xffffu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
    lo = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
    hi = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
}

__device__ __forceinline__ uint32_t f16x2_rn(float a, float b) {   // .x = a (low half)
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}
__device__ __forceinline__ float f16_lo_f(uint32_t p) { return __half2float(__ushort_as_half(static_cast<unsigned short>(p & 0xffffu))); }
__device__ __forceinline__ float f16_hi_f(uint32_t p) { return __half2float(__ushort_as_half(static_cast<unsigned short>(p >> 16))); }

template <int V>
__device__ __forceinline__ void tmem_ld_v(uint32_t taddr, uint32_t (&r)[V]) {
    if constexpr (V == 8) tc::tmem_ld8(taddr, r);
    else if constexpr (V == 16) tc::tmem_ld16(taddr, r);
    else tc::tmem_ld32(taddr, r);
}

// ------------------------------------------------------------------------------------------------
// Pieces shared by the split kernels
// ------------------------------------------------------------------------------------------------

// The query block of one head group: thread t holds head qh = 8 ((t >> 3) % (NH/8)) + (t & 7), dim
// groups qd0 + i (256/NH) (8 consecutive heads of one dim group per 8 lanes: conflict-free stores).
template <int NH>
struct QBlock {
    static constexpr int kPieces = NH * 64 / kMlaThreads;
    static constexpr int kStride = kMlaThreads / NH;
    int qh, qd0;
    bool real;
    uint4 v[kPieces];

    __device__ __forceinline__ void load(const uint16_t *q, int n, int n_heads, int h0, int nh_real, int tid) {
        qh = ((tid >> 3) % (NH / 8)) * 8 + (tid & 7);
        qd0 = (tid >> 3) / (NH / 8);
        real = qh < nh_real;
        const uint4 *qn = reinterpret_cast<const uint4 *>(q + (static_cast<int64_t>(n) * n_heads + h0 + (real ? qh : 0)) * kLatent);
#pragma unroll
        for (int i = 0; i < kPieces; i++) v[i] = real ? __ldg(qn + qd0 + i * kStride) : make_uint4(0u, 0u, 0u, 0u);
    }
    // largest |q| of the thread's pieces, as bf16 magnitude bits (ordered as integers)
    __device__ __forceinline__ unsigned absmax() const {
        unsigned mx = 0u;
#pragma unroll
        for (int i = 0; i < kPieces; i++) {
            const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int e = 0; e < 4; e++) mx = max(mx, max(w4[e] & 0x7fffu, (w4[e] >> 16) & 0x7fffu));
        }
        return mx;
    }
    // the block as fp16 core matrices (Qs: NH/8 x 64 x 128 B), each head scaled by the power of two
    // 2^e_h that puts its largest magnitude (qmax, every head's) in [2^14, 2^15) (exact: bf16
    // mantissas fit fp16), and the score factors qk[h] = sm_scale log2(e) 2^-e_h
    __device__ __forceinline__ void stage(const unsigned *qmax, float *qk, unsigned char *Qs, float sm_scale, int tid) const {
        const unsigned m = qmax[qh];
        int e = 0;
        if (m != 0u) {
            const int E = static_cast<int>(m >> 7) - 127;   // exponent of the largest magnitude
            e = min(120, max(-120, 14 - E));
        }
        const float f = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);   // 2^e, exact
        if (tid < NH) {
            const unsigned mt = qmax[tid];
            int et = 0;
            if (mt != 0u) et = min(120, max(-120, 14 - (static_cast<int>(mt >> 7) - 127)));
            qk[tid] = sm_scale * 1.4426950408889634f * __uint_as_float(static_cast<uint32_t>(127 - et) << 23);
        }
#pragma unroll
        for (int i = 0; i < kPieces; i++) {
            const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; k++)
                o[k] = f16x2_rn(__uint_as_float(w4[k] << 16) * f, __uint_as_float(w4[k] & 0xffff0000u) * f);
            const int dg = qd0 + i * kStride;
            *reinterpret_cast<uint4 *>(Qs + (qh >> 3) * 8192 + dg * 128 + (qh & 7) * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
};

// The codes of a chunk of ROWS cache rows in registers: every 16-byte piece of codes (and, for
// 4-bit rows, the two block scales of the piece) requested at once (piece P: row 8 rg + (P & 7),
// piece k of the row; eight lanes hold eight rows of one piece index, so that the widened lines
// they store are 128 contiguous bytes), then widened to an fp16 tile C[ROWS x 512] of 8x8 core
// matrices (row group rg at rg * 8192, dim group d at d * 128).
template <int ROWS, int kFmt>
struct RowTile {
    static constexpr bool kFp4 = kFmt == kFmtFp4;
    static constexpr int kRowB = kFp4 ? kFp4RowBytes : kRowBytes;      // bytes of a cache row
    static constexpr int kSclAt = kFp4 ? kFp4RowScaleAt : kLatent;     // where its fp32 row scale sits
    static constexpr int kPieces = kFp4 ? 16 : 32;                     // 16-byte pieces of codes in a row
    static constexpr int kCvt = ROWS * kPieces / kMlaThreads;
    uint4 gv[kCvt];
    uint32_t es[kFp4 ? kCvt : 1];

    __device__ __forceinline__ static void piece(int P, int &jl, int &rg, int &k) {
        const int klo = (P >> 3) & 3, rest = P >> 5;
        jl = P & 7;
        rg = rest % (ROWS / 8);
        k = (rest / (ROWS / 8)) * 4 + klo;
    }
    // ridx: the chunk's ROWS row indices (-1: no row)
    __device__ __forceinline__ void issue(const uint8_t *cache, const int *ridx, int tid) {
#pragma unroll
        for (int it = 0; it < kCvt; it++) {
            int jl, rg, k;
            piece(it * kMlaThreads + tid, jl, rg, k);
            const int r = ridx[rg * 8 + jl];
            const uint8_t *rp = cache + static_cast<int64_t>(r) * kRowB;
            gv[it] = r >= 0 ? __ldg(reinterpret_cast<const uint4 *>(rp) + k) : make_uint4(0u, 0u, 0u, 0u);
            if constexpr (kFp4)
                es[it] = r >= 0 ? __ldg(reinterpret_cast<const uint16_t *>(rp + kFp4ScalesAt) + k) : 0u;
        }
    }
    __device__ __forceinline__ static float row_scale(const uint8_t *cache, int r) {
        return r >= 0 ? __ldg(reinterpret_cast<const float *>(cache + static_cast<int64_t>(r) * kRowB + kSclAt)) : 0.0f;
    }
    __device__ __forceinline__ void convert(unsigned char *Cs, int tid) const {
#pragma unroll
        for (int it = 0; it < kCvt; it++) {
            int jl, rg, k;
            piece(it * kMlaThreads + tid, jl, rg, k);
            const uint4 w = gv[it];
            if constexpr (kFp4) {   // 32 codes: dim groups 4 k .. 4 k + 3 (block scales 2 k and 2 k + 1)
                const __half2_raw sc = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(es[it]), __NV_E4M3);
                const uint32_t s0 = static_cast<uint32_t>(sc.x) * 0x10001u, s1 = static_cast<uint32_t>(sc.y) * 0x10001u;
                uint32_t o0[4], o1[4], o2[4], o3[4];
                fp4_to_f16x8(w.x, s0, o0);
                fp4_to_f16x8(w.y, s0, o1);
                fp4_to_f16x8(w.z, s1, o2);
                fp4_to_f16x8(w.w, s1, o3);
                unsigned char *line = Cs + rg * 8192 + (4 * k) * 128 + jl * 16;
                *reinterpret_cast<uint4 *>(line) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
                *reinterpret_cast<uint4 *>(line + 128) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
                *reinterpret_cast<uint4 *>(line + 256) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
                *reinterpret_cast<uint4 *>(line + 384) = make_uint4(o3[0], o3[1], o3[2], o3[3]);
            } else {
                uint32_t o[8];
                if constexpr (kFmt == kFmtFp8) {
                    fp8_to_f16x4(w.x, o[0], o[1]);
                    fp8_to_f16x4(w.y, o[2], o[3]);
                    fp8_to_f16x4(w.z, o[4], o[5]);
                    fp8_to_f16x4(w.w, o[6], o[7]);
                } else {
                    codes_to_f16x4(w.x, o[0], o[1]);
                    codes_to_f16x4(w.y, o[2], o[3]);
                    codes_to_f16x4(w.z, o[4], o[5]);
                    codes_to_f16x4(w.w, o[6], o[7]);
                }
                unsigned char *line = Cs + rg * 8192 + (2 * k) * 128 + jl * 16;
                *reinterpret_cast<uint4 *>(line) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(line + 128) = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
    }
};

template <int ROWS, int NH, int kFmt>
__global__ void __launch_bounds__(kMlaThreads, 1) mla_split_tc_kernel(
    const uint16_t *__restrict__ q, int n_heads, const uint8_t *__restrict__ cache, int64_t n_rows,
    const int32_t *__restrict__ rows, int width, float sm_scale, int n_chunks, int n_hg,
    float *__restrict__ part_acc, float *__restrict__ part_ml, int *__restrict__ status, int early_q) {
    using L = MlaLayout<ROWS, NH>;
    constexpr int V = NH / 2;             // heads per softmax thread
    constexpr int kLboP = 32 * NH;        // P': bytes between row groups (2 NH / 8 head groups x 128 B)
    // early_q: the query block is an input no preceding kernel writes (the one-call step), so its
    // loads are issued before waiting for the preceding kernel; the row indices wait for it
    if (early_q) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    else pdl_begin();
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *Cs = smem + L::kC;
    unsigned char *Ps = smem + L::kP;
    unsigned char *Qs = smem + L::kQ;
    float *scl = reinterpret_cast<float *>(smem + L::kScl);
    int *ridx = reinterpret_cast<int *>(smem + L::kRow);
    float *red = reinterpret_cast<float *>(smem + L::kRed);
    float *red2 = reinterpret_cast<float *>(smem + L::kRed2);
    float *qk = reinterpret_cast<float *>(smem + L::kQk);
    unsigned *qmax = reinterpret_cast<unsigned *>(smem + L::kQmax);
    unsigned *words = reinterpret_cast<unsigned *>(smem + L::kWords);
    const uint32_t bar0 = tc::smem_addr(smem + L::kBar);
    const uint32_t bar_s = bar0, bar_o = bar0 + 8;

    const int n = blockIdx.y, c = blockIdx.x / n_hg, hg = blockIdx.x % n_hg;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h0 = hg * NH;
    const int nh_real = min(NH, n_heads - h0);
    const int64_t ml_base = (static_cast<int64_t>(n) * n_chunks + c) * n_heads + h0;
    GLM_TL(glm_tl_split, 0);
    GLM_TL_SMID(glm_tl_split);

    // 1. the query block's loads
    QBlock<NH> qb;
    qb.load(q, n, n_heads, h0, nh_real, tid);
    if (tid < NH) qmax[tid] = 0u;
    if (tid == 0) words[0] = 0u;
    if (early_q) asm volatile("griddepcontrol.wait;" ::: "memory");

    // 2. the chunk's row indices (entries past width or outside [0, n_rows) are padding)
    int myrow = -1;
    if (tid < ROWS) {
        const int j = c * ROWS + tid;
        const int r = j < width ? rows[static_cast<int64_t>(n) * width + j] : -1;
        myrow = (r >= 0 && r < n_rows) ? r : -1;
        ridx[tid] = myrow;
    }
    const int n_valid = __syncthreads_count(myrow >= 0);
    GLM_TL(glm_tl_split, 2);
    if (n_valid == 0) {   // no valid entry in this chunk: an empty partial
        if (tid < nh_real) {
            part_ml[2 * (ml_base + tid)] = -INFINITY;
            part_ml[2 * (ml_base + tid) + 1] = 0.0f;
        }
        return;
    }

    // 3. gather: every 16-byte piece of codes of the chunk's rows and every row scale requested at once
    RowTile<ROWS, kFmt> tile;
    tile.issue(cache, ridx, tid);
    const float my_scale = RowTile<ROWS, kFmt>::row_scale(cache, myrow);
    GLM_TL(glm_tl_split, 9);
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(&words[1]), 8 * NH);
        tc::tmem_relinquish();
        tc::fence_before_sync();
    }
    GLM_TL(glm_tl_split, 10);
    if (tid == 32) {
        tc::mbar_init(bar_s, 1);
        tc::mbar_init(bar_o, 1);
        tc::mbar_fence_init();
    }

    // 4. while the rows are in flight: the query block as fp16, each head scaled by the power of two
    //    2^e_h that puts its largest magnitude in [2^14, 2^15) (exact: bf16 mantissas fit fp16)
    const unsigned mx = qb.absmax();
    GLM_TL(glm_tl_split, 11);
    if (qb.real) atomicMax(&qmax[qb.qh], mx);
    __syncthreads();
    GLM_TL(glm_tl_split, 12);
    qb.stage(qmax, qk, Qs, sm_scale, tid);
    GLM_TL(glm_tl_split, 1);

    // 5. row scales, their maximum, and the codes widened to fp16 core matrices
    if (tid < ROWS) {
        scl[tid] = my_scale;
        const unsigned sm = __reduce_max_sync(0xffffffffu, __float_as_uint(my_scale));   // scales are >= 0
        if (lane == 0) atomicMax(&words[0], sm);
    }
    tile.convert(Cs, tid);
    GLM_TL(glm_tl_split, 3);
    tc::fence_proxy_async();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = words[1];
    bool ok;

    GLM_TL(glm_tl_split, 4);
    // 4. S^T = C . Q^T (M = ROWS rows, N = NH heads, K = 512)
    if (tid == 0) {
        const uint32_t idesc = tc::idesc_f16(ROWS, NH, false, false);
        const uint32_t ca = tc::smem_addr(Cs), qa = tc::smem_addr(Qs);
#pragma unroll 4
        for (int ks = 0; ks < kLatent / 16; ks++)
            tc::mma_bf16(tmem, tc::desc(ca + ks * 256, 128, 8192), tc::desc(qa + ks * 256, 128, 8192), idesc,
                         ks > 0 ? 1u : 0u);
        tc::mma_commit(bar_s);
    }
    ok = tc::mbar_wait(bar_s, 0, kMlaWaitLimit);
    if (!__syncthreads_and(ok)) {
        if (tid == 0) atomicOr(status, 1);
        tc::mbar_wait(bar_s, 0, kMlaWaitLimit);
        __syncthreads();
        goto done;
    }
    tc::fence_after_sync();
    GLM_TL(glm_tl_split, 5);

    // 5. softmax: warp w reads TMEM lane quadrant w % 4 (one row per lane) and heads [V (w / 4), +V)
    {
        const int quad = warp & 3, hh = warp >> 2;
        const int j = (ROWS == 128) ? quad * 32 + lane : (lane < 16 ? quad * 16 + lane : -1);
        uint32_t r[V];
        tmem_ld_v<V>(tmem + (static_cast<uint32_t>(quad * 32) << 16) + hh * V, r);
        tc::tmem_wait_ld();
        const bool rv = j >= 0 && ridx[j] >= 0;
        const float sc = rv ? scl[j] : 0.0f;
        float s[V], t[V];
#pragma unroll
        for (int i = 0; i < V; i++) {
            s[i] = rv ? __uint_as_float(r[i]) * sc * qk[hh * V + i] : -INFINITY;
            t[i] = s[i];
        }
        constexpr int kLow = (V == 32) ? 0 : (V == 16) ? 1 : 3;   // lane bits that repeat a head index
        constexpr int kShift = (V == 32) ? 0 : (V == 16) ? 1 : 2;
        float bm = butterfly<V, true>(t);
        if ((lane & kLow) == 0) red[quad * NH + hh * V + ((lane >> kShift) & (V - 1))] = bm;
        __syncthreads();
        const float smax = __uint_as_float(words[0]);
        const float ratio = rv ? __fdiv_rn(sc, smax) : 0.0f;   // scale_row / scale_max, in (0, 1]
#pragma unroll
        for (int i = 0; i < V; i++) {
            const int h = hh * V + i;
            const float m = fmaxf(fmaxf(red[h], red[NH + h]), fmaxf(red[2 * NH + h], red[3 * NH + h]));
            const float p = (rv && m != -INFINITY) ? exp2f(s[i] - m) : 0.0f;
            s[i] = p;
            t[i] = p;
        }
        float bl = butterfly<V, false>(t);
        if ((lane & kLow) == 0) red2[quad * NH + hh * V + ((lane >> kShift) & (V - 1))] = bl;
        if (j >= 0) {   // P' of this row as fp16 hi + lo, 8 heads per 16-byte line
#pragma unroll
            for (int g = 0; g < V / 8; g++) {
                uint32_t hi4[4], lo4[4];
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const float a = s[8 * g + 2 * e] * ratio, b = s[8 * g + 2 * e + 1] * ratio;
                    hi4[e] = f16x2_rn(a, b);
                    lo4[e] = f16x2_rn(a - f16_lo_f(hi4[e]), b - f16_hi_f(hi4[e]));
                }
                const int G = hh * (V / 8) + g;
                unsigned char *line = Ps + (j >> 3) * kLboP + G * 128 + (j & 7) * 16;
                *reinterpret_cast<uint4 *>(line) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                *reinterpret_cast<uint4 *>(line + (NH / 8) * 128) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
            }
        }
        tc::fence_before_sync();
    }
    tc::fence_proxy_async();
    __syncthreads();
    if (tid < nh_real) {   // (m, l) of each head, natural-log units
        const float m = fmaxf(fmaxf(red[tid], red[NH + tid]), fmaxf(red[2 * NH + tid], red[3 * NH + tid]));
        const float l = (red2[tid] + red2[NH + tid]) + (red2[2 * NH + tid] + red2[3 * NH + tid]);
        part_ml[2 * (ml_base + tid)] = m * 0.6931471805599453f;
        part_ml[2 * (ml_base + tid) + 1] = l;
    }

    GLM_TL(glm_tl_split, 6);
    // 6. O^T = C^T . P'^T (hi and lo heads side by side: N = 2 NH)
    if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_f16(128, 2 * NH, true, true);
        const uint32_t pa = tc::smem_addr(Ps), ca = tc::smem_addr(Cs);
#pragma unroll
        for (int ks = 0; ks < ROWS / 16; ks++) {
#pragma unroll
            for (int mt = 0; mt < kLatent / 128; mt++)
                tc::mma_bf16(tmem + mt * 2 * NH, tc::desc(ca + ks * 2 * 8192 + mt * 16 * 128, 8192, 128),
                             tc::desc(pa + ks * 2 * kLboP, kLboP, 128), idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar_o);
    }
    ok = tc::mbar_wait(bar_o, 0, kMlaWaitLimit);
    if (!__syncthreads_and(ok)) {
        if (tid == 0) atomicOr(status, 2);
        tc::mbar_wait(bar_o, 0, kMlaWaitLimit);
        __syncthreads();
        goto done;
    }
    tc::fence_after_sync();
    GLM_TL(glm_tl_split, 7);

    // 7. acc = scale_max (O_hi + O_lo): tile mt, lane quadrant q (latent dims 128 mt + 32 q + lane)
    {
        const int quad = warp & 3;
        const float smax = __uint_as_float(words[0]);
#pragma unroll 1
        for (int mt = warp >> 2; mt < kLatent / 128; mt += 2) {
            const int dim = mt * 128 + quad * 32 + lane;
            const uint32_t ta = tmem + (static_cast<uint32_t>(quad * 32) << 16) + mt * 2 * NH;
#pragma unroll 1
            for (int hb = 0; hb < NH; hb += 16) {
                uint32_t hi[16], lo[16];
                tc::tmem_ld16(ta + hb, hi);
                tc::tmem_ld16(ta + NH + hb, lo);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; e++)
                    if (hb + e < nh_real)
                        part_acc[(ml_base + hb + e) * kLatent + dim] =
                            smax * (__uint_as_float(hi[e]) + __uint_as_float(lo[e]));
            }
        }
    }
done:
    tc::fence_before_sync();
    __syncthreads();
    GLM_TL(glm_tl_split, 8);
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 8 * NH);
    }
}

// ------------------------------------------------------------------------------------------------
// Many queries: one CTA per (query, run of chunks, group of 64 heads) walks its chunks of 64
// entries with a running softmax state and the output accumulated in tensor memory, so that
// enough queries fill the SMs without cutting each query into per-chunk partials:
//   * the next chunk's rows are requested (and the indices of the one after it) before the
//     current chunk's work, so that their round trip hides behind it; its tile goes to the other
//     of two C buffers;
//   * S^T = C . Q^T as in the split kernel; per head the chunk's largest score m_c (log2 units);
//     the reference m_ref moves to m_c only when m_c > m_ref + 8, so exp2(s - m_ref) <= 2^8;
//   * the row-scale reference sigma (a power of two) moves to the next power of two >= the
//     chunk's largest row scale only when that exceeds 16 sigma;
//   * P' = exp2(s - m_ref) scale_row / sigma (<= 2^12) as an fp16 hi + lo pair, l = l alpha + sum
//     of exp2(s - m_ref) over the chunk's rows;
//   * when a reference moves, the accumulator is first multiplied in tensor memory by
//     alpha_h beta (alpha_h = exp2(m_ref,old - m_ref,new), beta = sigma_old / sigma_new);
//   * O^T += C^T . P'_hi^T + C^T . P'_lo^T into one accumulator of 4 tiles of 128 latent dims x 64
//     heads of tensor memory (the two terms as successive products, not side by side);
//   * at the end acc = sigma O with (m_ref ln 2, l) is one partial of the combine or, when the
//     CTA covers all of the query's entries, the combine's own result of one partial is written
//     directly (out = acc (1 / l), lse = m + log l).
// ------------------------------------------------------------------------------------------------
template <int NH>
struct MlaMultiLayout {
    static constexpr int kRows = 64;
    static constexpr int kCBytes = kRows * 1024;                      // one chunk's tile
    static constexpr int kC = 0;                                      // [2] tiles
    static constexpr int kQ = kC + 2 * kCBytes;                       // NH/8 x 64 x 128 B
    static constexpr int kPTerm = kRows * 2 * NH;                     // one term of P': 8 row groups x NH/8 head groups x 128 B
    static constexpr int kP = kQ + NH * 1024;                         // P' hi, then lo
    static constexpr int kScl = kP + 2 * kPTerm;                      // [2][64] row scales
    static constexpr int kRow = kScl + 2 * kRows * 4;                 // [2][64] row indices
    static constexpr int kRed = kRow + 2 * kRows * 4;                 // [4 quadrants][NH] partial maxima
    static constexpr int kRed2 = kRed + 4 * NH * 4;                   // [4][NH] partial sums
    static constexpr int kQk = kRed2 + 4 * NH * 4;                    // NH score factors
    static constexpr int kQmax = kQk + NH * 4;                        // NH |q| maxima (bf16 bits)
    static constexpr int kMref = kQmax + NH * 4;                      // NH reference maxima (log2 units)
    static constexpr int kLsum = kMref + NH * 4;                      // NH running sums
    static constexpr int kFac = kLsum + NH * 4;                       // NH factors of the accumulator
    static constexpr int kWords = kFac + NH * 4;                      // [0..1] chunk scale maxima (bits), [2] tmem base
    static constexpr int kBar = kWords + 16;                          // 2 mbarriers
    static constexpr int kBytes = kBar + 2 * 8;
    static_assert(kQ % 16 == 0 && kP % 16 == 0 && kBar % 8 == 0, "alignment");
    static_assert(kBytes <= 232448, "shared memory of one CTA");
};

// The smallest power of two >= x (1 for x <= 0, capped at 2^127).
__device__ __forceinline__ float pow2_ceil(float x) {
    if (!(x > 0.0f)) return 1.0f;
    const uint32_t b = __float_as_uint(x);
    int e = static_cast<int>(b >> 23) - 127;
    if ((b & 0x7fffffu) != 0u || e < -126) e += 1;
    e = max(-126, min(127, e));
    return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

template <int NH, int kFmt>
__global__ void __launch_bounds__(kMlaThreads, 1) mla_multi_tc_kernel(
    const uint16_t *__restrict__ q, int n_heads, const uint8_t *__restrict__ cache, int64_t n_rows,
    const int32_t *__restrict__ rows, int width, float sm_scale, int n_chunks, int cpc, int n_parts, int n_hg,
    float *__restrict__ part_acc, float *__restrict__ part_ml, uint16_t *__restrict__ out,
    float *__restrict__ out_f32, float *__restrict__ lse, int *__restrict__ status, int early_q) {
    using L = MlaMultiLayout<NH>;
    using Tile = RowTile<64, kFmt>;
    constexpr int ROWS = 64;
    constexpr int V = NH / 2;                                 // heads per softmax thread
    constexpr int kLboP = 16 * NH;                            // P': bytes between row groups
    constexpr uint32_t kSCol = 4 * NH;                        // S after the accumulator's 4 tiles
    constexpr int kCols = 5 * NH <= 256 ? 256 : 512;
    constexpr float kMaxGrow = 8.0f;
    constexpr int kLow = (V == 32) ? 0 : (V == 16) ? 1 : 3;   // lane bits that repeat a head index
    constexpr int kShift = (V == 32) ? 0 : (V == 16) ? 1 : 2;
    static_assert(NH % 32 == 0, "the accumulator is read and rescaled 32 heads at a time");
    if (early_q) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    else pdl_begin();
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *Cs = smem + L::kC;
    unsigned char *Ps = smem + L::kP;
    unsigned char *Qs = smem + L::kQ;
    float *scl = reinterpret_cast<float *>(smem + L::kScl);
    int *ridx = reinterpret_cast<int *>(smem + L::kRow);
    float *red = reinterpret_cast<float *>(smem + L::kRed);
    float *red2 = reinterpret_cast<float *>(smem + L::kRed2);
    float *qk = reinterpret_cast<float *>(smem + L::kQk);
    unsigned *qmax = reinterpret_cast<unsigned *>(smem + L::kQmax);
    float *mref = reinterpret_cast<float *>(smem + L::kMref);
    float *lsum = reinterpret_cast<float *>(smem + L::kLsum);
    float *fac = reinterpret_cast<float *>(smem + L::kFac);
    unsigned *words = reinterpret_cast<unsigned *>(smem + L::kWords);
    const uint32_t bar0 = tc::smem_addr(smem + L::kBar);
    const uint32_t bar_s = bar0, bar_o = bar0 + 8;

    const int n = blockIdx.y, pt = blockIdx.x / n_hg, hg = blockIdx.x % n_hg;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h0 = hg * NH;
    const int nh_real = min(NH, n_heads - h0);
    const int c0 = pt * cpc, c1 = min(n_chunks, c0 + cpc);
    const bool direct = out != nullptr;
    const int64_t ml_base = (static_cast<int64_t>(n) * n_parts + pt) * n_heads + h0;
    GLM_TL(glm_tl_split, 0);

    QBlock<NH> qb;
    qb.load(q, n, n_heads, h0, nh_real, tid);
    if (tid < NH) {
        qmax[tid] = 0u;
        mref[tid] = -INFINITY;
        lsum[tid] = 0.0f;
    }
    if (tid < 2) words[tid] = 0u;
    if (early_q) asm volatile("griddepcontrol.wait;" ::: "memory");

    // tid < ROWS: the row of entry c ROWS + tid (-1: none, past width, or outside [0, n_rows))
    auto row_of = [&](int c) -> int {
        const int j = c * ROWS + tid;
        if (tid >= ROWS || c >= c1 || j >= width) return -1;
        const int r = rows[static_cast<int64_t>(n) * width + j];
        return (r >= 0 && r < n_rows) ? r : -1;
    };
    const int r0 = row_of(c0);
    int r_next = row_of(c0 + 1);
    if (tid < ROWS) ridx[tid] = r0;
    int nv = __syncthreads_count(r0 >= 0);
    Tile tile;
    tile.issue(cache, ridx, tid);
    float my_scale = Tile::row_scale(cache, r0);
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(&words[2]), kCols);
        tc::tmem_relinquish();
        tc::fence_before_sync();
    }
    if (tid == 32) {
        tc::mbar_init(bar_s, 1);
        tc::mbar_init(bar_o, 1);
        tc::mbar_fence_init();
    }
    const unsigned mx = qb.absmax();
    if (qb.real) atomicMax(&qmax[qb.qh], mx);
    __syncthreads();
    qb.stage(qmax, qk, Qs, sm_scale, tid);
    if (tid < ROWS) {
        scl[tid] = my_scale;
        const unsigned sm = __reduce_max_sync(0xffffffffu, __float_as_uint(my_scale));   // scales are >= 0
        if (lane == 0) atomicMax(&words[0], sm);
    }
    tile.convert(Cs, tid);
    tc::fence_proxy_async();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = words[2];
    GLM_TL(glm_tl_split, 1);

    uint32_t s_phase = 0, o_phase = 0;   // commits issued on each barrier
    bool have_o = false;                 // the accumulator holds a chunk
    float sigma = 0.0f;                  // row-scale reference (0: none yet); the same in every thread
    float alpha = 1.0f;                  // tid < NH: this chunk's factor of l
    int fail = 0;
    const int quad = warp & 3, hh = warp >> 2;
    const int j = lane < 16 ? quad * 16 + lane : -1;   // the S row of this lane (M = 64: lanes 0-15 of a quadrant)

    for (int c = c0, i = 0; c < c1; c++, i++) {
        const int buf = i & 1;
        const bool more = c + 1 < c1;
        // a. the next chunk's indices and row requests; the indices of the chunk after it
        int nv_next = 0;
        if (more) {
            if (tid < ROWS) ridx[(buf ^ 1) * ROWS + tid] = r_next;
            if (tid == 0) words[buf ^ 1] = 0u;
            nv_next = __syncthreads_count(r_next >= 0);
            tile.issue(cache, ridx + (buf ^ 1) * ROWS, tid);
            my_scale = Tile::row_scale(cache, r_next);
            r_next = row_of(c + 2);
        }
        if (nv > 0) {
            // b. S^T = C . Q^T (M = 64 rows, N = NH heads, K = 512); its completion also means that
            //    every earlier accumulation has completed
            if (tid == 0) {
                tc::fence_after_sync();
                const uint32_t idesc = tc::idesc_f16(ROWS, NH, false, false);
                const uint32_t ca = tc::smem_addr(Cs + buf * L::kCBytes), qa = tc::smem_addr(Qs);
#pragma unroll 4
                for (int ks = 0; ks < kLatent / 16; ks++)
                    tc::mma_bf16(tmem + kSCol, tc::desc(ca + ks * 256, 128, 8192), tc::desc(qa + ks * 256, 128, 8192),
                                 idesc, ks > 0 ? 1u : 0u);
                tc::mma_commit(bar_s);
            }
            const bool ok = tc::mbar_wait(bar_s, s_phase & 1u, kMlaWaitLimit);
            s_phase++;
            if (!__syncthreads_and(ok)) {
                fail = 1;
                break;
            }
            tc::fence_after_sync();
            const float smax_c = __uint_as_float(words[buf]);
            const float sig_new = (sigma == 0.0f || smax_c > 16.0f * sigma) ? pow2_ceil(smax_c) : sigma;
            const float beta = sigma == 0.0f ? 1.0f : sigma / sig_new;   // powers of two: exact
            const float inv_sig = 1.0f / sig_new;

            // c. softmax: warp w reads TMEM lane quadrant w % 4 (row 16 (w % 4) + lane, lanes < 16)
            //    and heads [V (w / 4), +V)
            uint32_t r[V];
            tmem_ld_v<V>(tmem + (static_cast<uint32_t>(quad * 32) << 16) + kSCol + hh * V, r);
            tc::tmem_wait_ld();
            const bool rv = j >= 0 && ridx[buf * ROWS + j] >= 0;
            const float sc = rv ? scl[buf * ROWS + j] : 0.0f;
            float sv[V], t[V];
#pragma unroll
            for (int e = 0; e < V; e++) {
                sv[e] = rv ? __uint_as_float(r[e]) * sc * qk[hh * V + e] : -INFINITY;
                t[e] = sv[e];
            }
            const float bm = butterfly<V, true>(t);
            if ((lane & kLow) == 0) red[quad * NH + hh * V + ((lane >> kShift) & (V - 1))] = bm;
            __syncthreads();
            bool need = false;
            if (tid < NH) {
                const float mc = fmaxf(fmaxf(red[tid], red[NH + tid]), fmaxf(red[2 * NH + tid], red[3 * NH + tid]));
                const float mo = mref[tid];
                const float mn = (mo == -INFINITY || mc > mo + kMaxGrow) ? mc : mo;
                alpha = mo == -INFINITY ? 0.0f : exp2f(mo - mn);
                mref[tid] = mn;
                const float f = alpha * beta;
                fac[tid] = f;
                need = have_o && f != 1.0f;
            }
            const bool rescale = __syncthreads_or(need) != 0;
            sigma = sig_new;
            const float ratio = sc * inv_sig;   // scale_row / sigma (exact: sigma a power of two)
#pragma unroll
            for (int e = 0; e < V; e++) {
                const float m = mref[hh * V + e];
                const float pv = rv ? exp2f(sv[e] - m) : 0.0f;
                sv[e] = pv;
                t[e] = pv;
            }
            const float bl = butterfly<V, false>(t);
            if ((lane & kLow) == 0) red2[quad * NH + hh * V + ((lane >> kShift) & (V - 1))] = bl;
            if (j >= 0) {   // P' of this row as fp16 hi + lo, 8 heads per 16-byte line
#pragma unroll
                for (int g = 0; g < V / 8; g++) {
                    uint32_t hi4[4], lo4[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const float a = sv[8 * g + 2 * e] * ratio, b = sv[8 * g + 2 * e + 1] * ratio;
                        hi4[e] = f16x2_rn(a, b);
                        lo4[e] = f16x2_rn(a - f16_lo_f(hi4[e]), b - f16_hi_f(hi4[e]));
                    }
                    unsigned char *line = Ps + (j >> 3) * kLboP + (hh * (V / 8) + g) * 128 + (j & 7) * 16;
                    *reinterpret_cast<uint4 *>(line) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                    *reinterpret_cast<uint4 *>(line + L::kPTerm) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                }
            }
            if (rescale) {   // the accumulator times fac[h]: lane quadrant w % 4 of tiles w / 4 and w / 4 + 2
#pragma unroll 1
                for (int mt = hh; mt < 4; mt += 2) {
#pragma unroll 1
                    for (int cb = 0; cb < NH; cb += 32) {
                        const uint32_t ta = tmem + (static_cast<uint32_t>(quad * 32) << 16) + mt * NH + cb;
                        uint32_t a[32];
                        tc::tmem_ld32(ta, a);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e++) a[e] = __float_as_uint(__uint_as_float(a[e]) * fac[cb + e]);
                        tc::tmem_st32(ta, a);
                    }
                }
                tc::tmem_wait_st();
            }
            tc::fence_before_sync();
            tc::fence_proxy_async();
            __syncthreads();
            if (tid < NH)
                lsum[tid] = fmaf(lsum[tid], alpha, (red2[tid] + red2[NH + tid]) + (red2[2 * NH + tid] + red2[3 * NH + tid]));

            // d. O^T += C^T . P'_hi^T + C^T . P'_lo^T (M = 128 latent dims per tile, N = NH heads,
            //    K = 64 rows per term)
            if (tid == 0) {
                tc::fence_after_sync();
                const uint32_t idesc = tc::idesc_f16(128, NH, true, true);
                const uint32_t pa = tc::smem_addr(Ps), ca = tc::smem_addr(Cs + buf * L::kCBytes);
#pragma unroll
                for (int ks = 0; ks < ROWS / 16; ks++) {
#pragma unroll
                    for (int mt = 0; mt < kLatent / 128; mt++) {
                        const uint64_t da = tc::desc(ca + ks * 2 * 8192 + mt * 16 * 128, 8192, 128);
                        tc::mma_bf16(tmem + mt * NH, da, tc::desc(pa + ks * 2 * kLboP, kLboP, 128), idesc,
                                     (have_o || ks > 0) ? 1u : 0u);
                        tc::mma_bf16(tmem + mt * NH, da, tc::desc(pa + L::kPTerm + ks * 2 * kLboP, kLboP, 128), idesc, 1u);
                    }
                }
                tc::mma_commit(bar_o);
            }
            o_phase++;
            have_o = true;
        }
        // e. the next chunk's tile, into the buffer the accumulation of chunk c - 1 read (done: the
        //    S product of chunk c completed after it; with no S product, wait for it here)
        if (more) {
            if (nv == 0 && have_o) {
                const bool ok = tc::mbar_wait(bar_o, (o_phase - 1) & 1u, kMlaWaitLimit);
                if (!__syncthreads_and(ok)) {
                    fail = 2;
                    break;
                }
            }
            if (tid < ROWS) {
                scl[(buf ^ 1) * ROWS + tid] = my_scale;
                const unsigned sm = __reduce_max_sync(0xffffffffu, __float_as_uint(my_scale));
                if (lane == 0) atomicMax(&words[buf ^ 1], sm);
            }
            tile.convert(Cs + (buf ^ 1) * L::kCBytes, tid);
            tc::fence_proxy_async();
            __syncthreads();
        }
        nv = nv_next;
    }
    if (!fail && have_o) {
        const bool ok = tc::mbar_wait(bar_o, (o_phase - 1) & 1u, kMlaWaitLimit);
        if (!__syncthreads_and(ok)) fail = 2;
    }
    GLM_TL(glm_tl_split, 7);

    if (fail) {
        // a wait gave up: the status bit, bounded waits for this CTA's products still in flight,
        // and NaN outputs (direct) or a missing partial
        if (tid == 0) atomicOr(status, fail);
        if (s_phase > 0) tc::mbar_wait(bar_s, (s_phase - 1) & 1u, kMlaWaitLimit);
        if (o_phase > 0) tc::mbar_wait(bar_o, (o_phase - 1) & 1u, kMlaWaitLimit);
        if (direct) {
            for (int e = tid; e < nh_real * kLatent; e += kMlaThreads) {
                const int64_t ob = (static_cast<int64_t>(n) * n_heads + h0) * kLatent + e;
                out[ob] = 0x7fc0u;
                if (out_f32) out_f32[ob] = __int_as_float(0x7fc00000);
            }
            if (lse && tid < nh_real) lse[static_cast<int64_t>(n) * n_heads + h0 + tid] = __int_as_float(0x7fc00000);
        }
    } else if (!have_o) {
        // no valid entry: an empty partial, or the output of one (zeros, lse -inf)
        if (direct) {
            for (int e = tid; e < nh_real * kLatent; e += kMlaThreads) {
                const int64_t ob = (static_cast<int64_t>(n) * n_heads + h0) * kLatent + e;
                out[ob] = 0u;
                if (out_f32) out_f32[ob] = 0.0f;
            }
            if (lse && tid < nh_real) lse[static_cast<int64_t>(n) * n_heads + h0 + tid] = -INFINITY;
        } else if (tid < nh_real) {
            part_ml[2 * (ml_base + tid)] = -INFINITY;
            part_ml[2 * (ml_base + tid) + 1] = 0.0f;
        }
    } else {
        // acc = sigma O: tile mt, lane quadrant w % 4 (latent dim 128 mt + 32 (w % 4) + lane)
        tc::fence_after_sync();
#pragma unroll 1
        for (int mt = hh; mt < kLatent / 128; mt += 2) {
            const int dim = mt * 128 + quad * 32 + lane;
#pragma unroll 1
            for (int cb = 0; cb < NH; cb += 32) {
                uint32_t a[32];
                tc::tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + mt * NH + cb, a);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e++) {
                    const int h = cb + e;
                    if (h >= nh_real) break;
                    const float acc = sigma * __uint_as_float(a[e]);
                    if (direct) {
                        const float l = lsum[h];
                        const float v = acc * (l > 0.0f ? 1.0f / l : 0.0f);
                        const int64_t ob = (static_cast<int64_t>(n) * n_heads + h0 + h) * kLatent + dim;
                        out[ob] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                        if (out_f32) out_f32[ob] = v;
                    } else {
                        part_acc[(ml_base + h) * kLatent + dim] = acc;
                    }
                }
            }
        }
        if (tid < nh_real) {
            const float m = mref[tid] * 0.6931471805599453f, l = lsum[tid];
            if (direct) {
                if (lse) lse[static_cast<int64_t>(n) * n_heads + h0 + tid] = l > 0.0f ? m + logf(l) : -INFINITY;
            } else {
                part_ml[2 * (ml_base + tid)] = m;
                part_ml[2 * (ml_base + tid) + 1] = l;
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    GLM_TL(glm_tl_split, 8);
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kCols);
    }
}

int mla_tc_chunk() { return 64; }

long long mla_few_query_max(int n_heads, int num_sms) {
    const long long hg64 = (n_heads + 63) / 64;
    return (2ll * num_sms + hg64 - 1) / hg64 - 1;
}

MlaPlan mla_plan(int n_q, int n_heads, int width, int num_sms) {
    MlaPlan p{};
    p.rows = 64;
    p.n_chunks = (width + p.rows - 1) / p.rows;
    const long long hg64 = (n_heads + 63) / 64;
    const long long few_max = mla_few_query_max(n_heads, num_sms);
    if (n_q > few_max) {
        // many queries: the walking kernel, each query's entries in n_parts runs; the count that
        // minimises waves x (chunks per run + about two chunks of set-up and output), one run
        // (the output written directly, no combine) on ties; more than one run only while the
        // partials fit in what the largest few-query count needs (so that a workspace sized for
        // a count serves every smaller one)
        p.heads = 64;
        p.n_hg = static_cast<int>(hg64);
        p.multi = true;
        long long best = -1;
        for (int parts = 1; parts <= p.n_chunks; parts++) {
            const int cpc = (p.n_chunks + parts - 1) / parts;
            const int used = (p.n_chunks + cpc - 1) / cpc;
            if (used != parts) continue;
            if (parts > 1 && static_cast<long long>(n_q) * parts > few_max * p.n_chunks) break;
            const long long waves = (static_cast<long long>(n_q) * hg64 * parts + num_sms - 1) / num_sms;
            const long long cost = waves * (cpc + 2);
            if (best < 0 || cost < best) {
                best = cost;
                p.cpc = cpc;
                p.n_parts = parts;
            }
            if (waves > 64) break;
        }
        p.combine = p.n_parts > 1;
        return p;
    }
    // few queries: one CTA per 64-row chunk; 16 heads per CTA while they fill the SMs about one
    // and a half times, otherwise all 64 heads (no head group gathers a row another group of its
    // chunk gathers again)
    const long long ctas16 = static_cast<long long>(n_q) * p.n_chunks * ((n_heads + 15) / 16);
    p.heads = (2 * ctas16 <= 3ll * num_sms) ? 16 : 64;
    p.n_hg = (n_heads + p.heads - 1) / p.heads;
    p.cpc = 1;
    p.n_parts = p.n_chunks;
    p.multi = false;
    p.combine = true;
    return p;
}

template <int ROWS, int NH, int kFmt>
cudaError_t launch_t(const MlaPlan &p, const void *q, int n_heads, const uint8_t *cache, int64_t n_rows,
                     const int32_t *rows, int n_q, int width, float sm_scale, float *part_acc, float *part_ml,
                     int *status, cudaStream_t stream, bool early_q) {
    auto kernel = mla_split_tc_kernel<ROWS, NH, kFmt>;
    const int smem = MlaLayout<ROWS, NH>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kernel, dim3(p.n_chunks * p.n_hg, n_q), dim3(kMlaThreads), smem, stream,
                   static_cast<const uint16_t *>(q), n_heads, cache, n_rows, rows, width, sm_scale, p.n_chunks,
                   p.n_hg, part_acc, part_ml, status, early_q ? 1 : 0);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int kFmt>
cudaError_t launch_multi(const MlaPlan &p, const void *q, int n_heads, const uint8_t *cache, int64_t n_rows,
                         const int32_t *rows, int n_q, int width, float sm_scale, float *part_acc, float *part_ml,
                         void *out, float *out_f32, float *lse, int *status, cudaStream_t stream, bool early_q) {
    auto kernel = mla_multi_tc_kernel<64, kFmt>;
    const int smem = MlaMultiLayout<64>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const bool direct = !p.combine;
    e = launch_pdl(kernel, dim3(p.n_parts * p.n_hg, n_q), dim3(kMlaThreads), smem, stream,
                   static_cast<const uint16_t *>(q), n_heads, cache, n_rows, rows, width, sm_scale, p.n_chunks, p.cpc,
                   p.n_parts, p.n_hg, part_acc, part_ml, direct ? static_cast<uint16_t *>(out) : nullptr,
                   direct ? out_f32 : nullptr, direct ? lse : nullptr, status, early_q ? 1 : 0);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_mla_split_tc(const MlaPlan &p, const void *q, int n_heads, const int8_t *cache, int64_t n_rows,
                                const int32_t *rows, int n_q, int width, float sm_scale,
                                float *part_acc, float *part_ml, int *status, cudaStream_t stream, bool early_q,
                                int format, void *out, float *out_f32, float *lse) {
    const uint8_t *c8 = reinterpret_cast<const uint8_t *>(cache);
    if (p.multi) {
        if (!p.combine && !out) return cudaErrorInvalidValue;
        if (format == kFmtInt8)
            return launch_multi<kFmtInt8>(p, q, n_heads, c8, n_rows, rows, n_q, width, sm_scale, part_acc, part_ml, out,
                                          out_f32, lse, status, stream, early_q);
        if (format == kFmtFp8)
            return launch_multi<kFmtFp8>(p, q, n_heads, c8, n_rows, rows, n_q, width, sm_scale, part_acc, part_ml, out,
                                         out_f32, lse, status, stream, early_q);
        if (format == kFmtFp4)
            return launch_multi<kFmtFp4>(p, q, n_heads, c8, n_rows, rows, n_q, width, sm_scale, part_acc, part_ml, out,
                                         out_f32, lse, status, stream, early_q);
        return cudaErrorInvalidValue;
    }
#define GLM_MLA_LAUNCH(R, H, F)                                                                                  \
    if (p.rows == R && p.heads == H && format == F)                                                              \
        return launch_t<R, H, F>(p, q, n_heads, c8, n_rows, rows, n_q, width, sm_scale, part_acc, part_ml, status, \
                                 stream, early_q);
    GLM_MLA_LAUNCH(64, 16, kFmtInt8)
    GLM_MLA_LAUNCH(64, 64, kFmtInt8)
    GLM_MLA_LAUNCH(64, 16, kFmtFp8)
    GLM_MLA_LAUNCH(64, 64, kFmtFp8)
    GLM_MLA_LAUNCH(64, 16, kFmtFp4)
    GLM_MLA_LAUNCH(64, 64, kFmtFp4)
#undef GLM_MLA_LAUNCH
    return cudaErrorInvalidValue;
}

}  // namespace glm
