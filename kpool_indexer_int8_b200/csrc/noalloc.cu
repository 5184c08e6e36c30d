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
// the same data with the same plan, only the scratch lives here instead of in a caller buffer.
// The caller cannot read the scratch's status word, so a timed-out wait shows in the outputs
// instead: the combine then writes NaN to every output of the call.
#include "common.cuh"
#include "kernels.cuh"
#include "sparse_mla.cuh"

namespace {

// The scratch itself. Host code must not use this name as an address: on the host it only
// stands for the symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_mla_scratch[GLM_NOALLOC_SCRATCH_BYTES];

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" int glm_sparse_mla_decode_noalloc(const glm_dsa_dims *dims, const void *q,
                                             const int8_t *cache, int64_t n_rows,
                                             const int32_t *rows, int32_t n_q, int32_t width,
                                             float sm_scale, void *out, float *lse,
                                             float *out_f32, void *stream) {
    int rc = glm::abi::check_mla(dims, q, cache, n_rows, rows, n_q, width, sm_scale, out, lse, out_f32);
    if (rc != GLM_OK || n_q == 0) return rc;
    // size of this call's scratch, for the smallest chunk any plan uses; larger requests are
    // refused before anything is enqueued
    const int H = dims->n_heads;
    const int chunk = glm::mla_tc_chunk();
    const size_t parts = static_cast<size_t>(n_q) * static_cast<size_t>((width + chunk - 1) / chunk) *
                         static_cast<size_t>(H);
    const size_t acc_bytes = round256(parts * glm::kLatent * sizeof(float));
    const size_t ml_bytes = round256(parts * 2 * sizeof(float));
    if (acc_bytes + ml_bytes + 256 > GLM_NOALLOC_SCRATCH_BYTES) return GLM_ERR_WORKSPACE;

    // the scratch's device address on the current device, looked up on every call (a host-side
    // query; the first one on a device loads the library's device code there)
    void *base = nullptr;
    rc = glm::abi::cuda_status(cudaGetSymbolAddress(&base, g_mla_scratch));
    if (rc != GLM_OK) return rc;
    char *ws = static_cast<char *>(base);
    float *part_acc = reinterpret_cast<float *>(ws);
    float *part_ml = reinterpret_cast<float *>(ws + acc_bytes);
    int *status = reinterpret_cast<int *>(ws + acc_bytes + ml_bytes);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status word keeps the previous call's value: clear it for this call
    rc = glm::abi::cuda_status(cudaMemsetAsync(status, 0, sizeof(int), st));
    if (rc != GLM_OK) return rc;
    const glm::MlaPlan plan = glm::mla_plan(n_q, H, width, glm::abi::num_sms());
    rc = glm::abi::cuda_status(glm::launch_mla_split_tc(plan, q, H, cache, n_rows, rows, n_q, width, sm_scale,
                                                        part_acc, part_ml, status, st, false, 0, out, out_f32, lse));
    if (rc != GLM_OK || !plan.combine) return rc;   // (without a combine the kernel writes NaN itself on a give-up)
    return glm::abi::cuda_status(glm::launch_mla_combine(part_acc, part_ml, n_q, H, plan.n_parts, out, out_f32,
                                                         lse, st, status));
}
