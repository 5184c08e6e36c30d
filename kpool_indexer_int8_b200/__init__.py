"""Python binding of libglm_dsa.so, the C ABI of the GLM-5.3-Flash kpool DSA decode path (sm_100a).

Argument marshalling only: each function takes torch CUDA tensors, checks dtypes and shapes,
and calls the C entry point of the same name (include/glm_dsa.h) on the current torch stream.
Every step of the path runs in the library's CUDA kernels; there is no CPU fallback. Importing
this package without the built library raises ImportError (build it with
``python kpool_indexer_int8_b200/build.py``).
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libglm_dsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python kpool_indexer_int8_b200/build.py`")

lib = C.CDLL(LIB_PATH)

GLM_OK = 0
GLM_ERR_INVALID_ARG = -1
GLM_ERR_UNSUPPORTED = -2
GLM_ERR_WORKSPACE = -3
GLM_ERR_CUDA = -4
GLM_INVALID = -1
GLM_ROW_BYTES = 528
GLM_FP4_ROW_BYTES = 304
GLM_CACHE_INT8, GLM_CACHE_FP8, GLM_CACHE_FP4 = 0, 1, 2
GLM_OP_INDEX_SCORES_TOPK = 1
GLM_OP_TOPK_POOLS = 2
GLM_OP_SPARSE_MLA = 3
GLM_OP_DECODE_STEP = 4
GLM_PLAN_INDEX_MANY, GLM_PLAN_MLA_MANY, GLM_PLAN_MLA_COMBINE = 1, 2, 4

EXPORTS = ("glm_check_dims", "glm_status_string", "glm_last_cuda_error", "glm_kv_store_int8",
           "glm_kpool_build", "glm_kpool_build_q8", "glm_index_scores", "glm_index_scores_topk",
           "glm_index_topk_expand", "glm_index_topk_expand_q8",
           "glm_dsa_decode_step",
           "glm_topk_pools", "glm_expand_selection",
           "glm_sparse_mla_decode", "glm_dsa_workspace_size", "glm_kv_store_fp8", "glm_sparse_mla_decode_fp8",
           "glm_debug_set_cross_cta_wait_limit", "glm_mla_v_up", "glm_cp_candidates", "glm_merge_topk",
           "glm_lse_merge", "glm_kv_store_fp4", "glm_sparse_mla_decode_fp4", "glm_dsa_step_plan")


class glm_dsa_dims(C.Structure):
    """DsaDims of the pages ("Module glm5next_dsa_ref"): passed explicitly, never defaulted."""
    _fields_ = [("kv_lora_rank", C.c_int32), ("qk_rope_head_dim", C.c_int32),
                ("n_heads", C.c_int32), ("index_n_heads", C.c_int32),
                ("index_head_dim", C.c_int32), ("index_kpool", C.c_int32),
                ("index_topk", C.c_int32)]


class glm_dsa_step(C.Structure):
    """Arguments of glm_dsa_decode_step (every pointer a device pointer, None allowed where the
    C header allows NULL)."""
    _fields_ = [("latent_dev", C.c_void_p), ("slots_dev", C.c_void_p), ("n_new", C.c_int64),
                ("cache_dev", C.c_void_p), ("n_rows", C.c_int64),
                ("k_dev", C.c_void_p), ("gate_dev", C.c_void_p), ("ld_tokens", C.c_int64),
                ("ln_w_dev", C.c_void_p), ("ln_b_dev", C.c_void_p), ("ln_eps", C.c_float),
                ("pad_dev", C.c_void_p), ("len_dev", C.c_void_p), ("pool_begin_dev", C.c_void_p),
                ("batch", C.c_int32), ("max_new_pools", C.c_int32), ("pooled_dev", C.c_void_p),
                ("ld_pools", C.c_int64),
                ("q_idx_dev", C.c_void_p), ("w_dev", C.c_void_p), ("q_seq_dev", C.c_void_p),
                ("q_pos_dev", C.c_void_p), ("n_q", C.c_int32), ("select_k", C.c_int32),
                ("slot_map_dev", C.c_void_p), ("ld_slot", C.c_int64), ("out_width", C.c_int32),
                ("scores_dev", C.c_void_p), ("topk_dev", C.c_void_p), ("n_sel_dev", C.c_void_p),
                ("tok_dev", C.c_void_p), ("rows_dev", C.c_void_p),
                ("q_dev", C.c_void_p), ("sm_scale", C.c_float), ("out_dev", C.c_void_p),
                ("lse_dev", C.c_void_p), ("out_f32_dev", C.c_void_p),
                ("pooled_codes_dev", C.c_void_p), ("pooled_scales_dev", C.c_void_p), ("cache_format", C.c_int32),
                ("stop_after", C.c_int32)]


def make_dims(n_heads: int, kv_lora_rank: int = 512, qk_rope_head_dim: int = 0,
              index_n_heads: int = 32, index_head_dim: int = 128, index_kpool: int = 4,
              index_topk: int = 2048) -> glm_dsa_dims:
    return glm_dsa_dims(kv_lora_rank, qk_rope_head_dim, n_heads, index_n_heads, index_head_dim,
                        index_kpool, index_topk)


_P, _I64, _I32, _F32, _SZ = C.c_void_p, C.c_int64, C.c_int32, C.c_float, C.c_size_t
_D = C.POINTER(glm_dsa_dims)
lib.glm_check_dims.argtypes = [_D]
lib.glm_check_dims.restype = C.c_int
lib.glm_status_string.argtypes = [C.c_int]
lib.glm_status_string.restype = C.c_char_p
lib.glm_last_cuda_error.argtypes = []
lib.glm_last_cuda_error.restype = C.c_int
lib.glm_kv_store_int8.argtypes = [_D, _P, _P, _I64, _P, _I64, _P]
lib.glm_kv_store_int8.restype = C.c_int
lib.glm_kpool_build.argtypes = [_D, _P, _P, _I64, _P, _P, _F32, _P, _P, _P, _I32, _I32, _P, _I64, _P, _P]
lib.glm_kpool_build.restype = C.c_int
lib.glm_index_scores_topk.argtypes = [_D, _P, _P, _P, _I64, _P, _P, _P, _P, _I32, _I32, _I32, _P, _P,
                                      _P, _P, _SZ, _P]
lib.glm_index_scores_topk.restype = C.c_int
lib.glm_index_topk_expand.argtypes = [_D, _P, _P, _P, _I64, _P, _P, _P, _P, _I32, _I32, _I32, _P, _I64,
                                      _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]
lib.glm_index_topk_expand.restype = C.c_int
lib.glm_dsa_decode_step.argtypes = [_D, C.POINTER(glm_dsa_step), _P, _SZ, _P]
lib.glm_dsa_decode_step.restype = C.c_int
lib.glm_dsa_step_plan.argtypes = [_D, _I32, _I64, _I32, _I32, _I32, C.POINTER(C.c_int32), C.POINTER(C.c_int32)]
lib.glm_dsa_step_plan.restype = C.c_int
lib.glm_kpool_build_q8.argtypes = [_D, _P, _P, _I64, _P, _P, _F32, _P, _P, _P, _I32, _I32, _P, _P, _I64, _P, _P]
lib.glm_kpool_build_q8.restype = C.c_int
lib.glm_index_topk_expand_q8.argtypes = [_D, _P, _P, _P, _P, _I64, _P, _P, _P, _P, _I32, _I32, _I32, _P, _I64,
                                         _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]
lib.glm_index_topk_expand_q8.restype = C.c_int
lib.glm_index_scores.argtypes = [_D, _P, _P, _P, _I64, _P, _P, _P, _P, _I32, _I32, _P, _P]
lib.glm_index_scores.restype = C.c_int
lib.glm_topk_pools.argtypes = [_P, _I64, _P, _I32, _I32, _P, _P, _P, _SZ, _P]
lib.glm_topk_pools.restype = C.c_int
lib.glm_expand_selection.argtypes = [_D, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _P, _I64, _I32, _P,
                                     _P, _P]
lib.glm_expand_selection.restype = C.c_int
lib.glm_sparse_mla_decode.argtypes = [_D, _P, _P, _I64, _P, _I32, _I32, _F32, _P, _P, _P, _P, _SZ, _P]
lib.glm_sparse_mla_decode_fp8.argtypes = [_D, _P, _P, _I64, _P, _I32, _I32, _F32, _P, _P, _P, _P, _SZ, _P]
lib.glm_sparse_mla_decode_fp8.restype = C.c_int
lib.glm_kv_store_fp8.argtypes = [_D, _P, _P, _I64, _P, _I64, _P]
lib.glm_kv_store_fp8.restype = C.c_int
lib.glm_sparse_mla_decode_fp4.argtypes = [_D, _P, _P, _I64, _P, _I32, _I32, _F32, _P, _P, _P, _P, _SZ, _P]
lib.glm_sparse_mla_decode_fp4.restype = C.c_int
lib.glm_kv_store_fp4.argtypes = [_D, _P, _P, _I64, _P, _I64, _P]
lib.glm_kv_store_fp4.restype = C.c_int
lib.glm_sparse_mla_decode.restype = C.c_int
lib.glm_dsa_workspace_size.argtypes = [_D, _I32, _I32, _I64, _I32, _I32]
lib.glm_dsa_workspace_size.restype = C.c_size_t


class GlmError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = lib.glm_status_string(status).decode()
        if status == GLM_ERR_CUDA:
            msg += f" (cudaError {lib.glm_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [{status}]")
        self.status = status


def _check(status: int, what: str) -> None:
    if status != GLM_OK:
        raise GlmError(status, what)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _dev(t, dtype, name, ndim=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def check_dims(dims: glm_dsa_dims) -> int:
    return lib.glm_check_dims(C.byref(dims))


def glm_dsa_step_plan(dims, n_q, ld_pools, batch, width, int8_keys=False):
    """(kernels glm_dsa_decode_step enqueues, mask of GLM_PLAN_*) for a step of this shape."""
    k, f = C.c_int32(0), C.c_int32(0)
    _check(lib.glm_dsa_step_plan(C.byref(dims), n_q, ld_pools, batch, width, 1 if int8_keys else 0, C.byref(k),
                                 C.byref(f)), "glm_dsa_step_plan")
    return int(k.value), int(f.value)


def glm_dsa_workspace_size(dims, op, n_q, max_pools=0, select_k=1, width=1) -> int:
    v = lib.glm_dsa_workspace_size(C.byref(dims), op, n_q, max_pools, select_k, width)
    if v == C.c_size_t(-1).value:
        raise GlmError(GLM_ERR_INVALID_ARG, "glm_dsa_workspace_size")
    return int(v)


def glm_kv_store_int8(dims, latent, slots, cache, stream=None) -> None:
    """latent bf16 [n, 512], slots int64 [n], cache int8 [n_rows, 528] (or [blocks, 256, 528])."""
    _dev(latent, torch.bfloat16, "latent", 2)
    _dev(slots, torch.int64, "slots", 1)
    _dev(cache, torch.int8, "cache")
    n_rows = cache.numel() // GLM_ROW_BYTES
    _check(lib.glm_kv_store_int8(C.byref(dims), _ptr(latent), _ptr(slots), latent.shape[0],
                                 _ptr(cache), n_rows, _stream(stream)), "glm_kv_store_int8")


def glm_kv_store_fp8(dims, latent, slots, cache, stream=None) -> None:
    """The FP8 latent row: latent bf16 [n, 512], slots int64 [n], cache uint8 [n_rows, 528]."""
    _dev(latent, torch.bfloat16, "latent", 2)
    _dev(slots, torch.int64, "slots", 1)
    _dev(cache, torch.uint8, "cache")
    n_rows = cache.numel() // GLM_ROW_BYTES
    _check(lib.glm_kv_store_fp8(C.byref(dims), _ptr(latent), _ptr(slots), latent.shape[0],
                                _ptr(cache), n_rows, _stream(stream)), "glm_kv_store_fp8")


def glm_kv_store_fp4(dims, latent, slots, cache, stream=None) -> None:
    """The 4-bit latent row: latent bf16 [n, 512], slots int64 [n], cache uint8 [n_rows, 304]."""
    _dev(latent, torch.bfloat16, "latent", 2)
    _dev(slots, torch.int64, "slots", 1)
    _dev(cache, torch.uint8, "cache")
    n_rows = cache.numel() // GLM_FP4_ROW_BYTES
    _check(lib.glm_kv_store_fp4(C.byref(dims), _ptr(latent), _ptr(slots), latent.shape[0],
                                _ptr(cache), n_rows, _stream(stream)), "glm_kv_store_fp4")


def glm_kpool_build(dims, k, gate, ln_w, ln_b, ln_eps, pad, length, pooled, pool_begin=None,
                    max_new_pools=None, n_pools=None, stream=None) -> None:
    """k, gate bf16 [B, ld_tokens, 128]; ln_w, ln_b fp32 [128]; pad, length int32 [B];
    pooled fp32 [B, ld_pools, 128]; pool_begin int32 [B] or None; n_pools int32 [B] or None."""
    for t, dt, nm in ((k, torch.bfloat16, "k"), (gate, torch.bfloat16, "gate"),
                      (ln_w, torch.float32, "ln_w"), (ln_b, torch.float32, "ln_b"),
                      (pad, torch.int32, "pad"), (length, torch.int32, "len"),
                      (pooled, torch.float32, "pooled"), (pool_begin, torch.int32, "pool_begin"),
                      (n_pools, torch.int32, "n_pools")):
        _dev(t, dt, nm)
    B, ld_tokens = k.shape[0], k.shape[1]
    ld_pools = pooled.shape[1]
    if max_new_pools is None:
        max_new_pools = ld_pools
    _check(lib.glm_kpool_build(C.byref(dims), _ptr(k), _ptr(gate), ld_tokens, _ptr(ln_w), _ptr(ln_b),
                               float(ln_eps), _ptr(pad), _ptr(length), _ptr(pool_begin), B,
                               int(max_new_pools), _ptr(pooled), ld_pools, _ptr(n_pools),
                               _stream(stream)), "glm_kpool_build")


def glm_kpool_build_q8(dims, k, gate, ln_w, ln_b, ln_eps, pad, length, codes, scales, pool_begin=None,
                       max_new_pools=None, n_pools=None, stream=None) -> None:
    """The INT8 indexer state: codes int8 [B, ld_pools, 128], scales fp32 [B, ld_pools]; the other
    arguments as glm_kpool_build."""
    for t, dt, nm in ((k, torch.bfloat16, "k"), (gate, torch.bfloat16, "gate"),
                      (ln_w, torch.float32, "ln_w"), (ln_b, torch.float32, "ln_b"),
                      (pad, torch.int32, "pad"), (length, torch.int32, "len"),
                      (codes, torch.int8, "codes"), (scales, torch.float32, "scales"),
                      (pool_begin, torch.int32, "pool_begin"), (n_pools, torch.int32, "n_pools")):
        _dev(t, dt, nm)
    B, ld_tokens = k.shape[0], k.shape[1]
    ld_pools = codes.shape[1]
    if max_new_pools is None:
        max_new_pools = ld_pools
    _check(lib.glm_kpool_build_q8(C.byref(dims), _ptr(k), _ptr(gate), ld_tokens, _ptr(ln_w), _ptr(ln_b),
                                  float(ln_eps), _ptr(pad), _ptr(length), _ptr(pool_begin), B,
                                  int(max_new_pools), _ptr(codes), _ptr(scales), ld_pools, _ptr(n_pools),
                                  _stream(stream)), "glm_kpool_build_q8")


def glm_index_topk_expand_q8(dims, q_idx, w, codes, scales, q_seq, q_pos, pad, length, select_k, topk,
                             out_width, n_sel=None, slot_map=None, tok=None, rows=None, scores=None,
                             workspace=None, stream=None) -> None:
    """glm_index_topk_expand on the INT8 indexer state (codes int8 [B, ld_pools, 128], scales fp32
    [B, ld_pools])."""
    for t, dt, nm in ((q_idx, torch.bfloat16, "q_idx"), (w, torch.float32, "w"),
                      (codes, torch.int8, "codes"), (scales, torch.float32, "scales"),
                      (q_seq, torch.int32, "q_seq"), (q_pos, torch.int32, "q_pos"), (pad, torch.int32, "pad"),
                      (length, torch.int32, "len"), (topk, torch.int32, "topk"),
                      (n_sel, torch.int32, "n_sel"), (slot_map, torch.int64, "slot_map"),
                      (tok, torch.int32, "tok"), (rows, torch.int32, "rows"),
                      (scores, torch.float32, "scores"), (workspace, torch.uint8, "workspace")):
        _dev(t, dt, nm)
    ws_bytes = 0 if workspace is None else workspace.numel()
    ld_slot = 0 if slot_map is None else slot_map.shape[1]
    _check(lib.glm_index_topk_expand_q8(C.byref(dims), _ptr(q_idx), _ptr(w), _ptr(codes), _ptr(scales),
                                        codes.shape[1], _ptr(q_seq), _ptr(q_pos), _ptr(pad), _ptr(length),
                                        pad.shape[0], q_idx.shape[0], int(select_k), _ptr(slot_map), ld_slot,
                                        int(out_width), _ptr(scores), _ptr(topk), _ptr(n_sel), _ptr(tok),
                                        _ptr(rows), _ptr(workspace), ws_bytes, _stream(stream)),
           "glm_index_topk_expand_q8")


def glm_index_scores_topk(dims, q_idx, w, pooled, q_seq, q_pos, pad, length, select_k, topk,
                          n_sel=None, scores=None, workspace=None, stream=None) -> None:
    """q_idx bf16 [n_q, 32, 128], w fp32 [n_q, 32], pooled fp32 [B, ld_pools, 128];
    topk int32 [n_q, select_k]; scores fp32 [n_q, ld_pools] or None; workspace uint8 tensor."""
    for t, dt, nm in ((q_idx, torch.bfloat16, "q_idx"), (w, torch.float32, "w"),
                      (pooled, torch.float32, "pooled"), (q_seq, torch.int32, "q_seq"),
                      (q_pos, torch.int32, "q_pos"), (pad, torch.int32, "pad"),
                      (length, torch.int32, "len"), (topk, torch.int32, "topk"),
                      (n_sel, torch.int32, "n_sel"), (scores, torch.float32, "scores"),
                      (workspace, torch.uint8, "workspace")):
        _dev(t, dt, nm)
    n_q = q_idx.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel()
    _check(lib.glm_index_scores_topk(C.byref(dims), _ptr(q_idx), _ptr(w), _ptr(pooled), pooled.shape[1],
                                     _ptr(q_seq), _ptr(q_pos), _ptr(pad), _ptr(length), pad.shape[0],
                                     n_q, int(select_k), _ptr(scores), _ptr(topk), _ptr(n_sel),
                                     _ptr(workspace), ws_bytes, _stream(stream)),
           "glm_index_scores_topk")


def glm_index_topk_expand(dims, q_idx, w, pooled, q_seq, q_pos, pad, length, select_k, topk,
                          out_width, n_sel=None, slot_map=None, tok=None, rows=None, scores=None,
                          workspace=None, stream=None) -> None:
    """glm_index_scores_topk and glm_expand_selection in one launch: the arguments of both
    (tok / rows int32 [n_q, out_width], at least one; slot_map int64 [B, ld_slot] or None)."""
    for t, dt, nm in ((q_idx, torch.bfloat16, "q_idx"), (w, torch.float32, "w"),
                      (pooled, torch.float32, "pooled"), (q_seq, torch.int32, "q_seq"),
                      (q_pos, torch.int32, "q_pos"), (pad, torch.int32, "pad"),
                      (length, torch.int32, "len"), (topk, torch.int32, "topk"),
                      (n_sel, torch.int32, "n_sel"), (slot_map, torch.int64, "slot_map"),
                      (tok, torch.int32, "tok"), (rows, torch.int32, "rows"),
                      (scores, torch.float32, "scores"), (workspace, torch.uint8, "workspace")):
        _dev(t, dt, nm)
    ws_bytes = 0 if workspace is None else workspace.numel()
    ld_slot = 0 if slot_map is None else slot_map.shape[1]
    _check(lib.glm_index_topk_expand(C.byref(dims), _ptr(q_idx), _ptr(w), _ptr(pooled), pooled.shape[1],
                                     _ptr(q_seq), _ptr(q_pos), _ptr(pad), _ptr(length), pad.shape[0],
                                     q_idx.shape[0], int(select_k), _ptr(slot_map), ld_slot,
                                     int(out_width), _ptr(scores), _ptr(topk), _ptr(n_sel), _ptr(tok),
                                     _ptr(rows), _ptr(workspace), ws_bytes, _stream(stream)),
           "glm_index_topk_expand")


def glm_dsa_decode_step(dims, *, latent, slots, cache, k, gate, ln_w, ln_b, ln_eps, pad, length, pool_begin,
                        max_new_pools, pooled, q_idx, w, q_seq, q_pos, select_k, out_width, slot_map, rows,
                        topk, q, sm_scale, out, workspace, n_sel=None, tok=None, scores=None, lse=None,
                        out_f32=None, pooled_codes=None, pooled_scales=None, cache_format=GLM_CACHE_INT8,
                        stop_after=0, stream=None) -> None:
    """The whole step in one call: the arguments of glm_kv_store_int8, glm_kpool_build,
    glm_index_topk_expand and glm_sparse_mla_decode (same tensors and rules); with cache_format
    GLM_CACHE_FP8 / GLM_CACHE_FP4 the cache holds FP8 / 4-bit rows (uint8) and the step stores and
    attends as glm_kv_store_fp8 / _fp4 and glm_sparse_mla_decode_fp8 / _fp4. stop_after = k (1..3)
    runs only the step's first k kernels."""
    for t, dt, nm in ((latent, torch.bfloat16, "latent"), (slots, torch.int64, "slots"),
                      (cache, torch.int8 if cache_format == GLM_CACHE_INT8 else torch.uint8, "cache"),
                      (k, torch.bfloat16, "k"), (gate, torch.bfloat16, "gate"), (ln_w, torch.float32, "ln_w"),
                      (ln_b, torch.float32, "ln_b"), (pad, torch.int32, "pad"), (length, torch.int32, "len"),
                      (pool_begin, torch.int32, "pool_begin"), (pooled, torch.float32, "pooled"),
                      (q_idx, torch.bfloat16, "q_idx"), (w, torch.float32, "w"), (q_seq, torch.int32, "q_seq"),
                      (q_pos, torch.int32, "q_pos"), (slot_map, torch.int64, "slot_map"), (rows, torch.int32, "rows"),
                      (topk, torch.int32, "topk"), (q, torch.bfloat16, "q"), (out, torch.bfloat16, "out"),
                      (workspace, torch.uint8, "workspace"), (n_sel, torch.int32, "n_sel"), (tok, torch.int32, "tok"),
                      (scores, torch.float32, "scores"), (lse, torch.float32, "lse"), (out_f32, torch.float32, "out_f32"),
                      (pooled_codes, torch.int8, "pooled_codes"), (pooled_scales, torch.float32, "pooled_scales")):
        _dev(t, dt, nm)
    a = glm_dsa_step()
    v = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    a.latent_dev, a.slots_dev, a.n_new = v(latent), v(slots), slots.shape[0]
    a.cache_dev, a.n_rows = v(cache), cache.shape[0]
    a.k_dev, a.gate_dev, a.ld_tokens = v(k), v(gate), k.shape[1]
    a.ln_w_dev, a.ln_b_dev, a.ln_eps = v(ln_w), v(ln_b), float(ln_eps)
    a.pad_dev, a.len_dev, a.pool_begin_dev = v(pad), v(length), v(pool_begin)
    a.batch, a.max_new_pools = pad.shape[0], int(max_new_pools)
    a.pooled_dev, a.ld_pools = v(pooled), pooled.shape[1]
    a.q_idx_dev, a.w_dev, a.q_seq_dev, a.q_pos_dev = v(q_idx), v(w), v(q_seq), v(q_pos)
    a.n_q, a.select_k = q_idx.shape[0], int(select_k)
    a.slot_map_dev, a.ld_slot = v(slot_map), (0 if slot_map is None else slot_map.shape[1])
    a.out_width = int(out_width)
    a.scores_dev, a.topk_dev, a.n_sel_dev, a.tok_dev, a.rows_dev = v(scores), v(topk), v(n_sel), v(tok), v(rows)
    a.q_dev, a.sm_scale, a.out_dev = v(q), float(sm_scale), v(out)
    a.lse_dev, a.out_f32_dev = v(lse), v(out_f32)
    a.pooled_codes_dev, a.pooled_scales_dev = v(pooled_codes), v(pooled_scales)
    a.cache_format = int(cache_format)
    a.stop_after = int(stop_after)
    ws_bytes = 0 if workspace is None else workspace.numel()
    _check(lib.glm_dsa_decode_step(C.byref(dims), C.byref(a), _ptr(workspace), ws_bytes, _stream(stream)),
           "glm_dsa_decode_step")


def glm_index_scores(dims, q_idx, w, pooled, q_seq, q_pos, pad, length, scores, stream=None) -> None:
    """Scores only: scores fp32 [n_q, ld_pools] (entries past the visible pools are -inf)."""
    for t, dt, nm in ((q_idx, torch.bfloat16, "q_idx"), (w, torch.float32, "w"),
                      (pooled, torch.float32, "pooled"), (q_seq, torch.int32, "q_seq"),
                      (q_pos, torch.int32, "q_pos"), (pad, torch.int32, "pad"),
                      (length, torch.int32, "len"), (scores, torch.float32, "scores")):
        _dev(t, dt, nm)
    _check(lib.glm_index_scores(C.byref(dims), _ptr(q_idx), _ptr(w), _ptr(pooled), pooled.shape[1],
                                _ptr(q_seq), _ptr(q_pos), _ptr(pad), _ptr(length), pad.shape[0],
                                q_idx.shape[0], _ptr(scores), _stream(stream)), "glm_index_scores")


def glm_topk_pools(scores, n_visible, select_k, topk, n_sel=None, workspace=None, stream=None) -> None:
    """scores fp32 [n_q, ld_scores], n_visible int32 [n_q]; topk int32 [n_q, select_k]."""
    for t, dt, nm in ((scores, torch.float32, "scores"), (n_visible, torch.int32, "n_visible"),
                      (topk, torch.int32, "topk"), (n_sel, torch.int32, "n_sel"),
                      (workspace, torch.uint8, "workspace")):
        _dev(t, dt, nm)
    ws_bytes = 0 if workspace is None else workspace.numel()
    _check(lib.glm_topk_pools(_ptr(scores), scores.shape[1], _ptr(n_visible), scores.shape[0],
                              int(select_k), _ptr(topk), _ptr(n_sel), _ptr(workspace), ws_bytes,
                              _stream(stream)), "glm_topk_pools")


def glm_expand_selection(dims, topk, q_seq, q_pos, pad, length, out_width, n_sel=None,
                         slot_map=None, tok=None, rows=None, stream=None) -> None:
    """topk int32 [n_q, select_k]; slot_map int64 [B, ld_slot] or None;
    tok / rows int32 [n_q, out_width] (at least one)."""
    for t, dt, nm in ((topk, torch.int32, "topk"), (q_seq, torch.int32, "q_seq"),
                      (q_pos, torch.int32, "q_pos"), (pad, torch.int32, "pad"),
                      (length, torch.int32, "len"), (n_sel, torch.int32, "n_sel"),
                      (slot_map, torch.int64, "slot_map"), (tok, torch.int32, "tok"),
                      (rows, torch.int32, "rows")):
        _dev(t, dt, nm)
    ld_slot = 0 if slot_map is None else slot_map.shape[1]
    _check(lib.glm_expand_selection(C.byref(dims), _ptr(topk), _ptr(n_sel), _ptr(q_seq), _ptr(q_pos),
                                    _ptr(pad), _ptr(length), pad.shape[0], topk.shape[0],
                                    topk.shape[1], _ptr(slot_map), ld_slot, int(out_width),
                                    _ptr(tok), _ptr(rows), _stream(stream)), "glm_expand_selection")


def glm_sparse_mla_decode(dims, q, cache, rows, sm_scale, out, workspace, lse=None, out_f32=None,
                          stream=None) -> None:
    """q bf16 [n_q, n_heads, 512]; cache int8 [n_rows, 528]; rows int32 [n_q, width];
    out bf16 [n_q, n_heads, 512]; lse fp32 [n_q, n_heads] or None; out_f32 fp32 like out or None."""
    for t, dt, nm in ((q, torch.bfloat16, "q"), (cache, torch.int8, "cache"),
                      (rows, torch.int32, "rows"), (out, torch.bfloat16, "out"),
                      (workspace, torch.uint8, "workspace"), (lse, torch.float32, "lse"),
                      (out_f32, torch.float32, "out_f32")):
        _dev(t, dt, nm)
    n_rows = cache.numel() // GLM_ROW_BYTES
    _check(lib.glm_sparse_mla_decode(C.byref(dims), _ptr(q), _ptr(cache), n_rows, _ptr(rows),
                                     rows.shape[0], rows.shape[1], float(sm_scale), _ptr(out),
                                     _ptr(lse), _ptr(out_f32), _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "glm_sparse_mla_decode")


def glm_sparse_mla_decode_fp8(dims, q, cache, rows, sm_scale, out, workspace, lse=None, out_f32=None,
                              stream=None) -> None:
    """glm_sparse_mla_decode over FP8 rows: cache uint8 [n_rows, 528] (glm_kv_store_fp8)."""
    for t, dt, nm in ((q, torch.bfloat16, "q"), (cache, torch.uint8, "cache"),
                      (rows, torch.int32, "rows"), (out, torch.bfloat16, "out"),
                      (workspace, torch.uint8, "workspace"), (lse, torch.float32, "lse"),
                      (out_f32, torch.float32, "out_f32")):
        _dev(t, dt, nm)
    n_rows = cache.numel() // GLM_ROW_BYTES
    _check(lib.glm_sparse_mla_decode_fp8(C.byref(dims), _ptr(q), _ptr(cache), n_rows, _ptr(rows),
                                         rows.shape[0], rows.shape[1], float(sm_scale), _ptr(out),
                                         _ptr(lse), _ptr(out_f32), _ptr(workspace), workspace.numel(),
                                         _stream(stream)), "glm_sparse_mla_decode_fp8")


def glm_sparse_mla_decode_fp4(dims, q, cache, rows, sm_scale, out, workspace, lse=None, out_f32=None,
                              stream=None) -> None:
    """glm_sparse_mla_decode over 4-bit rows: cache uint8 [n_rows, 304] (glm_kv_store_fp4)."""
    for t, dt, nm in ((q, torch.bfloat16, "q"), (cache, torch.uint8, "cache"),
                      (rows, torch.int32, "rows"), (out, torch.bfloat16, "out"),
                      (workspace, torch.uint8, "workspace"), (lse, torch.float32, "lse"),
                      (out_f32, torch.float32, "out_f32")):
        _dev(t, dt, nm)
    n_rows = cache.numel() // GLM_FP4_ROW_BYTES
    _check(lib.glm_sparse_mla_decode_fp4(C.byref(dims), _ptr(q), _ptr(cache), n_rows, _ptr(rows),
                                         rows.shape[0], rows.shape[1], float(sm_scale), _ptr(out),
                                         _ptr(lse), _ptr(out_f32), _ptr(workspace), workspace.numel(),
                                         _stream(stream)), "glm_sparse_mla_decode_fp4")


# ------------------------------------------------------------------------------------------------
# allocation-free variant of the sparse MLA decode (for callers that cannot allocate a workspace)
# ------------------------------------------------------------------------------------------------
GLM_NOALLOC_SCRATCH_BYTES = 16 << 20
lib.glm_sparse_mla_decode_noalloc.argtypes = [_D, _P, _P, _I64, _P, _I32, _I32, _F32, _P, _P, _P, _P]
lib.glm_sparse_mla_decode_noalloc.restype = C.c_int


def glm_sparse_mla_decode_noalloc(dims, q, cache, rows, sm_scale, out, lse=None, out_f32=None,
                                  stream=None) -> None:
    """glm_sparse_mla_decode without a workspace: the split partials live in a fixed scratch inside
    the library (for callers that cannot allocate). Same tensors as glm_sparse_mla_decode."""
    for t, dt, nm in ((q, torch.bfloat16, "q"), (cache, torch.int8, "cache"),
                      (rows, torch.int32, "rows"), (out, torch.bfloat16, "out"),
                      (lse, torch.float32, "lse"), (out_f32, torch.float32, "out_f32")):
        _dev(t, dt, nm)
    n_rows = cache.numel() // GLM_ROW_BYTES
    _check(lib.glm_sparse_mla_decode_noalloc(C.byref(dims), _ptr(q), _ptr(cache), n_rows, _ptr(rows),
                                             rows.shape[0], rows.shape[1], float(sm_scale), _ptr(out),
                                             _ptr(lse), _ptr(out_f32), _stream(stream)),
           "glm_sparse_mla_decode_noalloc")


lib.glm_debug_set_cross_cta_wait_limit.argtypes = [C.c_uint32]
lib.glm_debug_set_cross_cta_wait_limit.restype = C.c_int
GLM_CROSS_CTA_WAIT_LIMIT = 1 << 21


def glm_debug_set_cross_cta_wait_limit(polls: int) -> None:
    """Polls before a wait of the fused index kernel's CTAs on one another gives up (tests only;
    GLM_CROSS_CTA_WAIT_LIMIT restores the default)."""
    _check(lib.glm_debug_set_cross_cta_wait_limit(int(polls)), "glm_debug_set_cross_cta_wait_limit")


lib.glm_mla_v_up.argtypes = [_D, _P, _P, _I32, _I32, _I32, _P, _P, _P]
lib.glm_mla_v_up.restype = C.c_int


def glm_mla_v_up(dims, o_lat, w_kv_b, qk_nope_head_dim, v_head_dim, out_v, out_v_f32=None, stream=None) -> None:
    """Up-projection of the latent attention output: o_lat bf16 [n_q, n_heads, 512], w_kv_b bf16
    [n_heads * (dk + dv), 512] -> out_v bf16 [n_q, n_heads, dv] (and fp32 if out_v_f32 is given)."""
    for t, dt, nm in ((o_lat, torch.bfloat16, "o_lat"), (w_kv_b, torch.bfloat16, "w_kv_b"),
                      (out_v, torch.bfloat16, "out_v"), (out_v_f32, torch.float32, "out_v_f32")):
        _dev(t, dt, nm)
    n_q = o_lat.shape[0]
    _check(lib.glm_mla_v_up(C.byref(dims), _ptr(o_lat), _ptr(w_kv_b), int(qk_nope_head_dim), int(v_head_dim), n_q,
                            _ptr(out_v), _ptr(out_v_f32), _stream(stream)), "glm_mla_v_up")


lib.glm_cp_candidates.argtypes = [_P, _I64, _P, _I32, _I32, _I32, _I32, _P, _P, _P]
lib.glm_cp_candidates.restype = C.c_int
lib.glm_merge_topk.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _P, _P, _P]
lib.glm_merge_topk.restype = C.c_int
lib.glm_lse_merge.argtypes = [_D, _P, _P, _I32, _I32, _P, _P, _P, _P]
lib.glm_lse_merge.restype = C.c_int


def glm_cp_candidates(scores, topk, rank, world, cand_scores, cand_ids, stream=None) -> None:
    """A rank's local selection as (score, global pool id) candidates: scores fp32 [n_q, ld], topk
    int32 [n_q, select_k] (local indices) -> cand_scores fp32 / cand_ids int32 [n_q, select_k]."""
    for t, dt, nm in ((scores, torch.float32, "scores"), (topk, torch.int32, "topk"),
                      (cand_scores, torch.float32, "cand_scores"), (cand_ids, torch.int32, "cand_ids")):
        _dev(t, dt, nm)
    _check(lib.glm_cp_candidates(_ptr(scores), scores.shape[1], _ptr(topk), topk.shape[0], topk.shape[1], int(rank),
                                 int(world), _ptr(cand_scores), _ptr(cand_ids), _stream(stream)), "glm_cp_candidates")


def glm_merge_topk(cand_scores, cand_ids, select_k, topk, n_sel=None, stream=None) -> None:
    """The global top-k of every part's candidates, laid out [n_parts, n_q, per_part]."""
    for t, dt, nm in ((cand_scores, torch.float32, "cand_scores"), (cand_ids, torch.int32, "cand_ids"),
                      (topk, torch.int32, "topk"), (n_sel, torch.int32, "n_sel")):
        _dev(t, dt, nm)
    n_parts, n_q, per = cand_ids.shape
    _check(lib.glm_merge_topk(_ptr(cand_scores), _ptr(cand_ids), n_parts, n_q, per, int(select_k), _ptr(topk),
                              _ptr(n_sel), _stream(stream)), "glm_merge_topk")


def glm_lse_merge(dims, out_parts, lse_parts, out, out_f32=None, lse=None, stream=None) -> None:
    """Log-sum-exp merge of attention parts: out_parts fp32 [n_parts, n_q, n_heads, 512], lse_parts
    fp32 [n_parts, n_q, n_heads] -> out bf16 [n_q, n_heads, 512] (fp32 copy and lse optional)."""
    for t, dt, nm in ((out_parts, torch.float32, "out_parts"), (lse_parts, torch.float32, "lse_parts"),
                      (out, torch.bfloat16, "out"), (out_f32, torch.float32, "out_f32"), (lse, torch.float32, "lse")):
        _dev(t, dt, nm)
    _check(lib.glm_lse_merge(C.byref(dims), _ptr(out_parts), _ptr(lse_parts), out_parts.shape[0], out_parts.shape[1],
                             _ptr(out), _ptr(out_f32), _ptr(lse), _stream(stream)), "glm_lse_merge")
