"""One decode (or prefill-chunk) step of the kpool DSA path as a sequence of C-ABI calls.

Order of the steps follows the pages ("GLM-5.3 Kernels" README: store_int8 then the sparse MLA
over indexer-selected rows; "Module glm5next_dsa_ref": pool_states -> index_scores ->
topk_pools -> expand_selection -> masked attention):

    glm_kv_store_int8 -> glm_kpool_build -> glm_index_scores_topk -> glm_expand_selection
      -> glm_sparse_mla_decode

A step runs as one call (glm_dsa_decode_step: the store, the pool build, the fused scoring +
selection + expansion and the sparse attention in four kernels); run_stages issues the
separate calls, for checking each stage on its own. This module only owns device buffers (allocated with torch) and marshals them into the calls;
all arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import (GLM_CACHE_FP4, GLM_CACHE_FP8, GLM_CACHE_INT8, GLM_FP4_ROW_BYTES, GLM_OP_DECODE_STEP,
               GLM_OP_INDEX_SCORES_TOPK, GLM_OP_SPARSE_MLA, GLM_ROW_BYTES, glm_dsa_decode_step, glm_dsa_workspace_size,
               glm_expand_selection, glm_index_scores_topk, glm_index_topk_expand, glm_index_topk_expand_q8,
               glm_kpool_build, glm_kpool_build_q8, glm_kv_store_fp4, glm_kv_store_fp8, glm_kv_store_int8,
               glm_sparse_mla_decode, glm_sparse_mla_decode_fp4, glm_sparse_mla_decode_fp8, make_dims)

LATENT = 512
IDX_HEADS = 32
IDX_DIM = 128
KPOOL = 4


@dataclass
class DecodeBuffers:
    """Device tensors of one step. State (cache, pooled, k, gate) persists across steps."""
    dims: object
    select_k: int
    out_width: int
    sm_scale: float
    ln_eps: float
    # resident state
    cache: torch.Tensor      # int8 [n_rows, 528]
    pooled: torch.Tensor     # fp32 [B, ld_pools, 128]
    k: torch.Tensor          # bf16 [B, ld_tokens, 128]
    gate: torch.Tensor       # bf16 [B, ld_tokens, 128]
    ln_w: torch.Tensor       # fp32 [128]
    ln_b: torch.Tensor       # fp32 [128]
    pad: torch.Tensor        # int32 [B]
    len: torch.Tensor        # int32 [B]
    slot_map: torch.Tensor   # int64 [B, ld_tokens]
    # per-step inputs
    new_latent: torch.Tensor  # bf16 [n_new, 512]
    new_slots: torch.Tensor   # int64 [n_new]
    pool_begin: torch.Tensor  # int32 [B]
    max_new_pools: int
    q_idx: torch.Tensor      # bf16 [n_q, 32, 128]
    w: torch.Tensor          # fp32 [n_q, 32]
    q: torch.Tensor          # bf16 [n_q, Hm, 512]
    q_seq: torch.Tensor      # int32 [n_q]
    q_pos: torch.Tensor      # int32 [n_q]
    # outputs and scratch
    topk: torch.Tensor       # int32 [n_q, select_k]
    n_sel: torch.Tensor      # int32 [n_q]
    tok: torch.Tensor        # int32 [n_q, out_width]
    rows: torch.Tensor       # int32 [n_q, out_width]
    out: torch.Tensor        # bf16 [n_q, Hm, 512]
    lse: torch.Tensor        # fp32 [n_q, Hm]
    ws_index: torch.Tensor   # uint8 workspace
    ws_mla: torch.Tensor     # uint8 workspace
    ws_step: torch.Tensor    # uint8 workspace of the one-call step
    scores: Optional[torch.Tensor] = None  # fp32 [n_q, ld_pools] when requested
    out_f32: Optional[torch.Tensor] = None
    pooled_codes: Optional[torch.Tensor] = None   # INT8 indexer state: int8 [B, ld_pools, 128]
    pooled_scales: Optional[torch.Tensor] = None  #                       fp32 [B, ld_pools]
    fp8: bool = False                             # the cache holds FP8 rows (uint8)
    fp4: bool = False                             # the cache holds 4-bit rows (uint8 [n_rows, 304])

    @property
    def cache_format(self) -> int:
        return GLM_CACHE_FP4 if self.fp4 else GLM_CACHE_FP8 if self.fp8 else GLM_CACHE_INT8


def allocate(n_heads: int, batch: int, ld_tokens: int, n_rows: int, n_q: int, n_new: int,
             select_k: int, out_width: int, sm_scale: float, ln_eps: float, max_new_pools: int,
             device, keep_scores: bool = False, keep_f32: bool = False, q8: bool = False,
             fp8: bool = False, fp4: bool = False) -> DecodeBuffers:
    dims = make_dims(n_heads)
    ld_pools = max(1, ld_tokens // KPOOL)
    f = dict(device=device)
    ws_i = glm_dsa_workspace_size(dims, GLM_OP_INDEX_SCORES_TOPK, n_q, ld_pools, select_k)
    ws_m = glm_dsa_workspace_size(dims, GLM_OP_SPARSE_MLA, n_q, width=out_width)
    ws_s = glm_dsa_workspace_size(dims, GLM_OP_DECODE_STEP, n_q, ld_pools, select_k, out_width)
    return DecodeBuffers(
        dims=dims, select_k=select_k, out_width=out_width, sm_scale=sm_scale, ln_eps=ln_eps,
        cache=torch.zeros(n_rows, GLM_FP4_ROW_BYTES if fp4 else GLM_ROW_BYTES,
                          dtype=torch.uint8 if (fp8 or fp4) else torch.int8, **f),
        fp8=fp8, fp4=fp4,
        pooled=torch.zeros(batch, ld_pools, IDX_DIM, dtype=torch.float32, **f),
        k=torch.zeros(batch, ld_tokens, IDX_DIM, dtype=torch.bfloat16, **f),
        gate=torch.zeros(batch, ld_tokens, IDX_DIM, dtype=torch.bfloat16, **f),
        ln_w=torch.zeros(IDX_DIM, dtype=torch.float32, **f),
        ln_b=torch.zeros(IDX_DIM, dtype=torch.float32, **f),
        pad=torch.zeros(batch, dtype=torch.int32, **f),
        len=torch.zeros(batch, dtype=torch.int32, **f),
        slot_map=torch.full((batch, ld_tokens), -1, dtype=torch.int64, **f),
        new_latent=torch.zeros(n_new, LATENT, dtype=torch.bfloat16, **f),
        new_slots=torch.full((n_new,), -1, dtype=torch.int64, **f),
        pool_begin=torch.zeros(batch, dtype=torch.int32, **f),
        max_new_pools=max_new_pools,
        q_idx=torch.zeros(n_q, IDX_HEADS, IDX_DIM, dtype=torch.bfloat16, **f),
        w=torch.zeros(n_q, IDX_HEADS, dtype=torch.float32, **f),
        q=torch.zeros(n_q, n_heads, LATENT, dtype=torch.bfloat16, **f),
        q_seq=torch.zeros(n_q, dtype=torch.int32, **f),
        q_pos=torch.zeros(n_q, dtype=torch.int32, **f),
        topk=torch.full((n_q, select_k), -1, dtype=torch.int32, **f),
        n_sel=torch.zeros(n_q, dtype=torch.int32, **f),
        tok=torch.full((n_q, out_width), -1, dtype=torch.int32, **f),
        rows=torch.full((n_q, out_width), -1, dtype=torch.int32, **f),
        out=torch.zeros(n_q, n_heads, LATENT, dtype=torch.bfloat16, **f),
        lse=torch.zeros(n_q, n_heads, dtype=torch.float32, **f),
        ws_index=torch.empty(max(ws_i, 1), dtype=torch.uint8, **f),
        ws_mla=torch.empty(max(ws_m, 1), dtype=torch.uint8, **f),
        ws_step=torch.empty(max(ws_s, 1), dtype=torch.uint8, **f),
        scores=torch.empty(n_q, ld_pools, dtype=torch.float32, **f) if keep_scores else None,
        out_f32=torch.empty(n_q, n_heads, LATENT, dtype=torch.float32, **f) if keep_f32 else None,
        pooled_codes=torch.zeros(batch, ld_pools, IDX_DIM, dtype=torch.int8, **f) if q8 else None,
        pooled_scales=torch.zeros(batch, ld_pools, dtype=torch.float32, **f) if q8 else None,
    )


def store(b: DecodeBuffers, stream=None) -> None:
    if b.fp4:
        glm_kv_store_fp4(b.dims, b.new_latent, b.new_slots, b.cache, stream=stream)
        return
    if b.fp8:
        glm_kv_store_fp8(b.dims, b.new_latent, b.new_slots, b.cache, stream=stream)
        return
    glm_kv_store_int8(b.dims, b.new_latent, b.new_slots, b.cache, stream=stream)


def build_pools(b: DecodeBuffers, length=None, pool_begin=None, max_new_pools=None, stream=None) -> None:
    if b.pooled_codes is not None:
        glm_kpool_build_q8(b.dims, b.k, b.gate, b.ln_w, b.ln_b, b.ln_eps, b.pad,
                           b.len if length is None else length, b.pooled_codes, b.pooled_scales,
                           pool_begin=b.pool_begin if pool_begin is None else pool_begin,
                           max_new_pools=b.max_new_pools if max_new_pools is None else max_new_pools,
                           stream=stream)
        return
    glm_kpool_build(b.dims, b.k, b.gate, b.ln_w, b.ln_b, b.ln_eps, b.pad,
                    b.len if length is None else length, b.pooled,
                    pool_begin=b.pool_begin if pool_begin is None else pool_begin,
                    max_new_pools=b.max_new_pools if max_new_pools is None else max_new_pools,
                    stream=stream)


def index_topk(b: DecodeBuffers, stream=None) -> None:
    glm_index_scores_topk(b.dims, b.q_idx, b.w, b.pooled, b.q_seq, b.q_pos, b.pad, b.len,
                          b.select_k, b.topk, n_sel=b.n_sel, scores=b.scores,
                          workspace=b.ws_index, stream=stream)


def expand(b: DecodeBuffers, stream=None) -> None:
    glm_expand_selection(b.dims, b.topk, b.q_seq, b.q_pos, b.pad, b.len, b.out_width,
                         n_sel=b.n_sel, slot_map=b.slot_map, tok=b.tok, rows=b.rows, stream=stream)


def index_topk_expand(b: DecodeBuffers, stream=None) -> None:
    if b.pooled_codes is not None:
        glm_index_topk_expand_q8(b.dims, b.q_idx, b.w, b.pooled_codes, b.pooled_scales, b.q_seq, b.q_pos, b.pad,
                                 b.len, b.select_k, b.topk, b.out_width, n_sel=b.n_sel, slot_map=b.slot_map,
                                 tok=b.tok, rows=b.rows, scores=b.scores, workspace=b.ws_index, stream=stream)
        return
    glm_index_topk_expand(b.dims, b.q_idx, b.w, b.pooled, b.q_seq, b.q_pos, b.pad, b.len, b.select_k,
                          b.topk, b.out_width, n_sel=b.n_sel, slot_map=b.slot_map, tok=b.tok, rows=b.rows,
                          scores=b.scores, workspace=b.ws_index, stream=stream)


def attend(b: DecodeBuffers, stream=None) -> None:
    if b.fp4:
        glm_sparse_mla_decode_fp4(b.dims, b.q, b.cache, b.rows, b.sm_scale, b.out, b.ws_mla, lse=b.lse,
                                  out_f32=b.out_f32, stream=stream)
        return
    if b.fp8:
        glm_sparse_mla_decode_fp8(b.dims, b.q, b.cache, b.rows, b.sm_scale, b.out, b.ws_mla, lse=b.lse,
                                  out_f32=b.out_f32, stream=stream)
        return
    glm_sparse_mla_decode(b.dims, b.q, b.cache, b.rows, b.sm_scale, b.out, b.ws_mla, lse=b.lse,
                          out_f32=b.out_f32, stream=stream)


STAGES = (("store_int8", store), ("kpool_build", build_pools), ("index_topk_expand", index_topk_expand),
          ("sparse_mla_decode", attend))


def run_stages(b: DecodeBuffers, stream=None) -> None:
    """One whole step as the separate calls, in order, on one stream."""
    for _, fn in STAGES:
        fn(b, stream=stream)


def run_step(b: DecodeBuffers, stream=None, stop_after: int = 0) -> None:
    """One whole step through the one-call entry point (stop_after = k: its first k kernels only)."""
    glm_dsa_decode_step(b.dims, latent=b.new_latent, slots=b.new_slots, cache=b.cache, k=b.k, gate=b.gate,
                        ln_w=b.ln_w, ln_b=b.ln_b, ln_eps=b.ln_eps, pad=b.pad, length=b.len,
                        pool_begin=b.pool_begin, max_new_pools=b.max_new_pools, pooled=b.pooled, q_idx=b.q_idx,
                        w=b.w, q_seq=b.q_seq, q_pos=b.q_pos, select_k=b.select_k, out_width=b.out_width,
                        slot_map=b.slot_map, rows=b.rows, topk=b.topk, q=b.q, sm_scale=b.sm_scale, out=b.out,
                        workspace=b.ws_step, n_sel=b.n_sel, tok=b.tok, scores=b.scores, lse=b.lse,
                        out_f32=b.out_f32, pooled_codes=b.pooled_codes, pooled_scales=b.pooled_scales,
                        cache_format=b.cache_format, stop_after=stop_after, stream=stream)
