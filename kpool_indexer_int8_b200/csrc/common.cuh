// common.cuh -- small device helpers shared by the kernels of the kpool DSA decode path.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "glm_dsa.h"

// Phase stamps of a timeline build (compiled with -DGLM_TIMELINE; they compile to nothing
// otherwise): thread t of a CTA records %globaltimer into slot k of the CTA's row of a per-kernel
// table, read back through <table>_read(host buffer of 2048 x 16 uint64).
#ifdef GLM_TIMELINE
#define GLM_TL_TABLE(name)                                                            \
    __device__ unsigned long long name[2048][16];                                     \
    extern "C" int name##_read(void *h) { return (int)cudaMemcpyFromSymbol(h, name, sizeof(name)); }
#define GLM_TL_AT(name, k, t)                                                         \
    do {                                                                              \
        if (threadIdx.x == (t)) {                                                     \
            unsigned long long t_;                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_)::"memory");          \
            name[(blockIdx.y * gridDim.x + blockIdx.x) & 2047][k] = t_;               \
        }                                                                             \
    } while (0)
#define GLM_TL_SMID(name)                                                             \
    do {                                                                              \
        if (threadIdx.x == 0) {                                                       \
            unsigned s_;                                                              \
            asm volatile("mov.u32 %0, %%smid;" : "=r"(s_));                          \
            name[(blockIdx.y * gridDim.x + blockIdx.x) & 2047][15] = s_;              \
        }                                                                             \
    } while (0)
#else
#define GLM_TL_TABLE(name)
#define GLM_TL_AT(name, k, t) \
    do {                      \
    } while (0)
#define GLM_TL_SMID(name) \
    do {                  \
    } while (0)
#endif
#define GLM_TL(name, k) GLM_TL_AT(name, k, 0)

namespace glm {

constexpr int kLatent = 512;        // kv_lora_rank
constexpr int kRowBytes = 528;      // 512 codes + fp32 scale + 12 zero bytes
constexpr int kFp4RowBytes = 304;   // 256 code pairs + 32 E4M3 block scales + fp32 row scale + 12 zero bytes
constexpr int kFp4ScalesAt = 256;   // the block scales (one per 16 values)
constexpr int kFp4RowScaleAt = 288; // the row scale
// The latent cache row formats: int8 codes, E4M3 codes (both 528 bytes, one fp32 scale), and
// block-scaled E2M1 codes (304 bytes).
enum CacheFormat { kFmtInt8 = 0, kFmtFp8 = 1, kFmtFp4 = 2 };
constexpr int kIdxHeads = 32;       // indexer heads
constexpr int kIdxDim = 128;        // indexer head dim
constexpr int kKpool = 4;           // tokens per pool
constexpr int kMaxSelect = 2048;    // largest select_k the top-k kernel sorts on chip
constexpr int kMaxHeads = 128;      // largest n_heads of the MLA kernels

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Reduce V values per lane (V a power of two <= 32) across the warp's 32 lanes with max (kMax) or
// sum: halving steps hand half of the values to the partner lane, so that after log2(V) steps lane
// l holds value index (l >> (5 - log2 V)) & (V - 1), reduced over the lanes that differ from l in
// the bits already used; the remaining steps finish the reduction over the other bits. Returns the
// lane's value (every lane with the same index holds the same result).
template <int V, bool kMax>
__device__ __forceinline__ float butterfly(float (&v)[V]) {
    const int lane = threadIdx.x & 31;
    auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
#pragma unroll
    for (int half = V / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < half; i++) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, bit));
        }
    }
    float r = v[0];
    constexpr int kRest = (V == 32) ? 0 : (V == 16) ? 1 : (V == 8) ? 2 : (V == 4) ? 3 : (V == 2) ? 4 : 5;
#pragma unroll
    for (int k = 0; k < kRest; k++) r = op(r, __shfl_xor_sync(0xffffffffu, r, 1 << (kRest - 1 - k)));
    return r;
}

// Order-preserving map of an fp32 score to an unsigned key (larger score -> larger key);
// -0.0 is folded onto +0.0 first so that the two compare equal.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s == 0.0f ? 0.0f : s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Number of pools visible to a query at q_pos of a sequence (pad, len): complete pools whose
// four slots are all at or before q_pos, capped at the pooled-key buffer's capacity.
__device__ __forceinline__ int visible_pools(int pad, int len, int q_pos, long long ld_pools) {
    int upto = q_pos - pad + 1;
    if (upto < 0) upto = 0;
    int n = min(len, upto) / kKpool;
    if (len < 0) n = 0;
    return static_cast<int>(min(static_cast<long long>(n), ld_pools));
}

// Programmatic dependent launch: a kernel launched with launch_pdl may start while the previous
// kernel of the stream is still running; pdl_begin() makes it wait (before any global memory
// access) until that kernel has finished and its writes are visible, then lets the next kernel
// of the stream be scheduled. Without the launch attribute both instructions are no-ops.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(std::forward<Args>(args))...);
}

}  // namespace glm
