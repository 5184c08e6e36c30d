// noalloc.cu -- the sparse NoPE MLA decode without a workspace argument.
//
// Some callers cannot allocate device memory at the point where they run the attention: plugin
// interfaces of inference engines that hand a kernel only its input and output tensors (no
// workspace), and serving loops that forbid any allocation after start-up so that their memory
// footprint stays fixed. For them this file keeps the split-KV scratch (per-chunk partial
// accumulators, their softmax maxima and sums, and a status word) in one fixed array compiled
// into the library. Every GPU that loads the library holds this array until the process exits.
//
// The computation is exactly glm_sparse_mla_decode's: the same split and combine kernels run on
// the same data, only the scratch lives here instead of in a caller buffer.
#include <mutex>

#include "common.cuh"
#include "sparse_mla.cuh"

namespace {

// The scratch itself. Host code must not use this name as an address: on the host it only
// stands for the symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_mla_scratch[GLM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Device address of the scratch on the current device, looked up once per device.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_mla_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

int noalloc_cuda_status(cudaError_t e) { return e == cudaSuccess ? GLM_OK : GLM_ERR_CUDA; }

}  // namespace

extern "C" int glm_sparse_mla_decode_noalloc(const glm_dsa_dims *dims, const void *q,
                                             const int8_t *cache, int64_t n_rows,
                                             const int32_t *rows, int32_t n_q, int32_t width,
                                             float sm_scale, void *out, float *lse,
                                             float *out_f32, void *stream) {
    int rc = glm_check_dims(dims);
    if (rc != GLM_OK) return rc;
    if (n_q < 0 || n_rows < 0 || width < 1 || width > 65536 || n_q > 65535) return GLM_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale)) return GLM_ERR_INVALID_ARG;
    if (n_q == 0) return GLM_OK;
    if (!q || !rows || !out || (n_rows > 0 && !cache)) return GLM_ERR_INVALID_ARG;
    const uintptr_t a16 = 15;
    if ((reinterpret_cast<uintptr_t>(q) & a16) || (cache && (reinterpret_cast<uintptr_t>(cache) & a16)) ||
        (reinterpret_cast<uintptr_t>(rows) & 3) || (reinterpret_cast<uintptr_t>(out) & a16) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) || (out_f32 && (reinterpret_cast<uintptr_t>(out_f32) & a16)))
        return GLM_ERR_INVALID_ARG;
    // size of this call's scratch; larger requests are refused before anything is enqueued
    const int H = dims->n_heads;
    const int chunk = glm::mla_tc_chunk();
    const int n_chunks = (width + chunk - 1) / chunk;
    const size_t parts = static_cast<size_t>(n_q) * static_cast<size_t>(n_chunks) * static_cast<size_t>(H);
    const size_t acc_bytes = round256(parts * glm::kLatent * sizeof(float));
    const size_t ml_bytes = round256(parts * 2 * sizeof(float));
    if (acc_bytes + ml_bytes + 256 > GLM_NOALLOC_SCRATCH_BYTES) return GLM_ERR_WORKSPACE;

    void *base = nullptr;
    rc = noalloc_cuda_status(scratch_address(&base));
    if (rc != GLM_OK) return rc;
    char *ws = static_cast<char *>(base);
    float *part_acc = reinterpret_cast<float *>(ws);
    float *part_ml = reinterpret_cast<float *>(ws + acc_bytes);
    int *status = reinterpret_cast<int *>(ws + acc_bytes + ml_bytes);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status word keeps the previous call's value: clear it for this call
    rc = noalloc_cuda_status(cudaMemsetAsync(status, 0, sizeof(int), st));
    if (rc != GLM_OK) return rc;
    rc = noalloc_cuda_status(glm::launch_mla_split_tc(q, H, cache, n_rows, rows, n_q, width, sm_scale,
                                                      part_acc, part_ml, status, st));
    if (rc != GLM_OK) return rc;
    return noalloc_cuda_status(glm::launch_mla_combine(part_acc, part_ml, n_q, H, n_chunks, out, out_f32,
                                                       lse, st));
}
