// expand.cu -- selected pools -> token indices and cache rows ("Module glm5next_dsa_ref",
// expand_selection and trap 6: expand selected pools into raw token indices, append the visible
// tail, pad with INVALID; all out_width entries are written).
//
// Grid (ceil(out_width / 256), n_q): one thread per output entry. Entry j < 4*n_sel is token pad + 4*topk[j/4] + j%4; the next `tail`
// entries are pad + 4*n_vis .. q_pos; the rest are -1. The cache row of each token comes from
// the sequence's slot map (or is the token itself without one).
#include "common.cuh"

namespace glm {

constexpr int kExpandThreads = 256;

__global__ void __launch_bounds__(kExpandThreads) expand_kernel(
    const int32_t *__restrict__ topk, const int32_t *__restrict__ n_sel_in,
    const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos,
    const int32_t *__restrict__ pad, const int32_t *__restrict__ len, int batch, int select_k,
    const int64_t *__restrict__ slot_map, int64_t ld_slot, int out_width,
    int32_t *__restrict__ tok_out, int32_t *__restrict__ rows_out) {
    pdl_begin();
    __shared__ int s_nsel;
    const int n = blockIdx.y;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t base = static_cast<int64_t>(n) * out_width;
    const int b = q_seq[n];
    if (b < 0 || b >= batch) {  // outside the contract: the whole row is -1
        if (j < out_width) {
            if (tok_out) tok_out[base + j] = GLM_INVALID;
            if (rows_out) rows_out[base + j] = GLM_INVALID;
        }
        return;
    }
    const int pb = pad[b], qp = q_pos[n];
    const int n_vis = visible_pools(pb, len[b], qp, 0x7fffffffll);
    const int32_t *tk = topk + static_cast<int64_t>(n) * select_k;
    if (threadIdx.x == 0) s_nsel = n_sel_in ? n_sel_in[n] : select_k;
    __syncthreads();
    if (!n_sel_in) {  // the list ends at its first -1
        for (int i = threadIdx.x; i < select_k; i += blockDim.x)
            if (tk[i] < 0) atomicMin(&s_nsel, i);
        __syncthreads();
    }
    const int n_sel = max(0, min(min(s_nsel, select_k), n_vis));
    const int last = min(qp, pb + len[b] - 1);  // the tail stops at the query or the sequence end
    const int tail = max(0, last - (pb + kKpool * n_vis) + 1);
    const int n_valid = kKpool * n_sel + tail;
    if (j < out_width) {
        int t = GLM_INVALID;
        if (j < kKpool * n_sel) {
            const int p = tk[j / kKpool];
            if (p >= 0 && p < n_vis) t = pb + kKpool * p + (j % kKpool);
        } else if (j < n_valid) {
            t = pb + kKpool * n_vis + (j - kKpool * n_sel);
        }
        if (tok_out) tok_out[base + j] = t;
        if (rows_out) {
            int r = t;
            if (slot_map) {
                r = GLM_INVALID;
                if (t >= 0 && t < ld_slot) {
                    const int64_t v = slot_map[static_cast<int64_t>(b) * ld_slot + t];
                    r = (v >= 0 && v <= 0x7fffffffll) ? static_cast<int>(v) : GLM_INVALID;
                }
            }
            rows_out[base + j] = r;
        }
    }
}

cudaError_t launch_expand(const int32_t *topk, const int32_t *n_sel, const int32_t *q_seq,
                          const int32_t *q_pos, const int32_t *pad, const int32_t *len, int batch,
                          int n_q, int select_k, const int64_t *slot_map, int64_t ld_slot, int out_width,
                          int32_t *tok, int32_t *rows, cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>((out_width + kExpandThreads - 1) / kExpandThreads), n_q);
    launch_pdl(expand_kernel, dim3(grid), dim3(kExpandThreads), 0, stream, topk, n_sel, q_seq, q_pos, pad, len, batch, select_k,
                                                      slot_map, ld_slot, out_width, tok, rows);
    return cudaGetLastError();
}

}  // namespace glm
