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

template <int ROWS, int NH, int kFmt>
__global__ void __launch_bounds__(kMlaThreads, 1) mla_split_tc_kernel(
    const uint16_t *__restrict__ q, int n_heads, const uint8_t *__restrict__ cache, int64_t n_rows,
    const int32_t *__restrict__ rows, int width, float sm_scale, int n_chunks, int n_hg,
    float *__restrict__ part_acc, float *__restrict__ part_ml, int *__restrict__ status, int early_q) {
    using L = MlaLayout<ROWS, NH>;
    constexpr bool kFp4 = kFmt == kFmtFp4;
    constexpr int kRowB = kFp4 ? kFp4RowBytes : kRowBytes;      // bytes of a cache row
    constexpr int kSclAt = kFp4 ? kFp4RowScaleAt : kLatent;     // where its fp32 row scale sits
    constexpr int kPieces = kFp4 ? 16 : 32;                     // 16-byte pieces of codes in a row
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

    // 1. the query block's loads: thread t holds head qh = 8 ((t >> 3) % (NH/8)) + (t & 7), dim
    //    groups qd0 + i (256/NH) (8 consecutive heads of one dim group per 8 lanes: conflict-free stores)
    constexpr int kQPieces = NH * 64 / kMlaThreads;
    constexpr int kQStride = kMlaThreads / NH;
    const int qh = ((tid >> 3) % (NH / 8)) * 8 + (tid & 7);
    const int qd0 = (tid >> 3) / (NH / 8);
    const bool qreal = qh < nh_real;
    if (tid < NH) qmax[tid] = 0u;
    if (tid == 0) words[0] = 0u;
    uint4 qv[kQPieces];
    {
        const uint4 *qn = reinterpret_cast<const uint4 *>(q + (static_cast<int64_t>(n) * n_heads + h0 + (qreal ? qh : 0)) * kLatent);
#pragma unroll
        for (int i = 0; i < kQPieces; i++) qv[i] = qreal ? __ldg(qn + qd0 + i * kQStride) : make_uint4(0u, 0u, 0u, 0u);
    }
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

    // 3. gather: every 16-byte piece of codes of the chunk's rows (and, for 4-bit rows, the two
    //    block scales of the piece) and every row scale is requested at once (piece P: row
    //    8 rg + (P & 7), piece k of the row; eight lanes hold eight rows of one piece index, so
    //    that the widened lines they store are 128 contiguous bytes)
    constexpr int kCvt = ROWS * kPieces / kMlaThreads;
    uint4 gv[kCvt];
    uint32_t es[kFp4 ? kCvt : 1];
#pragma unroll
    for (int it = 0; it < kCvt; it++) {
        const int P = it * kMlaThreads + tid;
        const int jl = P & 7, klo = (P >> 3) & 3, rest = P >> 5;
        const int rg = rest % (ROWS / 8), k = (rest / (ROWS / 8)) * 4 + klo;
        const int r = ridx[rg * 8 + jl];
        const uint8_t *rp = cache + static_cast<int64_t>(r) * kRowB;
        gv[it] = r >= 0 ? __ldg(reinterpret_cast<const uint4 *>(rp) + k) : make_uint4(0u, 0u, 0u, 0u);
        if constexpr (kFp4)
            es[it] = r >= 0 ? __ldg(reinterpret_cast<const uint16_t *>(rp + kFp4ScalesAt) + k) : 0u;
    }
    const float my_scale = myrow >= 0 ? __ldg(reinterpret_cast<const float *>(cache + static_cast<int64_t>(myrow) * kRowB + kSclAt)) : 0.0f;
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
    unsigned mx = 0u;   // largest |q| of the thread's pieces, as bf16 magnitude bits (ordered as integers)
#pragma unroll
    for (int i = 0; i < kQPieces; i++) {
        const uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
        for (int e = 0; e < 4; e++) mx = max(mx, max(w4[e] & 0x7fffu, (w4[e] >> 16) & 0x7fffu));
    }
    GLM_TL(glm_tl_split, 11);
    if (qreal) atomicMax(&qmax[qh], mx);
    __syncthreads();
    GLM_TL(glm_tl_split, 12);
    {
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
        for (int i = 0; i < kQPieces; i++) {
            const uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; k++)
                o[k] = f16x2_rn(__uint_as_float(w4[k] << 16) * f, __uint_as_float(w4[k] & 0xffff0000u) * f);
            const int dg = qd0 + i * kQStride;
            *reinterpret_cast<uint4 *>(Qs + (qh >> 3) * 8192 + dg * 128 + (qh & 7) * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    GLM_TL(glm_tl_split, 1);

    // 5. row scales, their maximum, and the codes widened to fp16 core matrices
    if (tid < ROWS) {
        scl[tid] = my_scale;
        const unsigned sm = __reduce_max_sync(0xffffffffu, __float_as_uint(my_scale));   // scales are >= 0
        if (lane == 0) atomicMax(&words[0], sm);
    }
#pragma unroll
    for (int it = 0; it < kCvt; it++) {
        const int P = it * kMlaThreads + tid;
        const int jl = P & 7, klo = (P >> 3) & 3, rest = P >> 5;
        const int rg = rest % (ROWS / 8), k = (rest / (ROWS / 8)) * 4 + klo;
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
            continue;
        }
        uint32_t o[8];
        if (kFmt == kFmtFp8) {
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

int mla_tc_chunk() { return 64; }

MlaPlan mla_plan(int n_q, int n_heads, int width, int num_sms) {
    // 64-row chunks of 16 heads while they fill the SMs about one and a half times; otherwise
    // 64-row chunks of all 64 heads (no head group gathers a row another group of its chunk
    // gathers again)
    MlaPlan p{};
    const long long ctas16 = static_cast<long long>(n_q) * ((width + 63) / 64) * ((n_heads + 15) / 16);
    p.rows = 64;
    p.heads = (2 * ctas16 <= 3ll * num_sms) ? 16 : 64;
    p.n_chunks = (width + p.rows - 1) / p.rows;
    p.n_hg = (n_heads + p.heads - 1) / p.heads;
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

cudaError_t launch_mla_split_tc(const MlaPlan &p, const void *q, int n_heads, const int8_t *cache, int64_t n_rows,
                                const int32_t *rows, int n_q, int width, float sm_scale,
                                float *part_acc, float *part_ml, int *status, cudaStream_t stream, bool early_q,
                                int format) {
    const uint8_t *c8 = reinterpret_cast<const uint8_t *>(cache);
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
