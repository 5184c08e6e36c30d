"""Context parallelism: one sequence's decode over several ranks (one process per GPU).

TensorFold issue #402, 'Credit': tokens are interleaved over the ranks, local candidates are
merged into the global top-k, and attention partials are merged by log-sum-exp in rank order. The
unit here is the pool (its four tokens stay together, so each rank can pool its own keys):

  * rank r of `world` holds pools p = r + world * i at local index i (its pooled keys), the cache
    rows of their tokens, and the visible tail (the tokens past the last complete pool) when it
    would own the next pool;
  * each rank scores and selects among its own visible pools (glm_index_scores_topk over a local
    pseudo-sequence of that many pools), turns the selection into (score, global pool id)
    candidates (glm_cp_candidates), and the ranks all-gather them;
  * every rank runs the same merge (glm_merge_topk) -- exactly the selection over all pools, since
    each globally selected pool is among its own rank's select_k best -- and expands it
    (glm_expand_selection) through its own slot map, so that the tokens it does not hold map to -1;
  * each rank attends over its own rows (glm_sparse_mla_decode), the ranks all-gather
    (out, lse), and every rank merges them in rank order (glm_lse_merge): identical outputs on
    every rank.

The arithmetic runs in the library's kernels; this module owns the index bookkeeping and the two
all-gathers (any torch.distributed group: NCCL over NVLink between GPUs, gloo in the CPU tests of the
bookkeeping). No TMA multicast is involved: peer data arrives by the collective into local memory.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (GLM_OP_INDEX_SCORES_TOPK, GLM_OP_SPARSE_MLA, glm_cp_candidates, glm_dsa_workspace_size,
               glm_expand_selection, glm_index_scores_topk, glm_lse_merge, glm_merge_topk,
               glm_sparse_mla_decode)

KPOOL = 4


def pool_owner(p: int, world: int) -> int:
    """The rank that holds pool p."""
    return p % world


def local_index(p: int, world: int) -> int:
    """Where pool p sits among its rank's pools."""
    return p // world


def local_pool_count(n_pools: int, rank: int, world: int) -> int:
    """How many of pools 0 .. n_pools - 1 rank holds."""
    return max(0, (n_pools - rank + world - 1) // world)


def token_owner(pad: int, length: int, t: int, world: int) -> int:
    """The rank that holds padded token t of a sequence (pad, length): its pool's rank; tokens of
    the incomplete last pool (the tail) go to the rank of that pool."""
    return pool_owner((t - pad) // KPOOL, world)


def owns_token(pad: int, length: int, t: int, rank: int, world: int) -> bool:
    return pad <= t < pad + length and token_owner(pad, length, t, world) == rank


@dataclass
class CpShard:
    """One rank's share of one sequence (batch 1): pooled keys of its pools at local indices,
    its cache rows, and a slot map from every padded token to its local cache row (-1 elsewhere)."""
    rank: int
    world: int
    pooled: torch.Tensor       # fp32 [1, ld_local, 128]
    cache: torch.Tensor        # int8 [n_rows_local, 528]
    slot_map: torch.Tensor     # int64 [1, ld_tokens]
    pad: int
    length: int


def cp_decode(dims, shard: CpShard, q_idx, w, q, q_pos: int, select_k: int, out_width: int, sm_scale: float,
              all_gather, stream=None):
    """One decode query of a context-parallel sequence on this rank. ``all_gather(t)`` returns the
    [world, *t.shape] stack of every rank's t in rank order (torch.distributed.all_gather_into_tensor
    on a group, or a stand-in that calls the same code for every rank). Returns (out bf16, out_f32,
    lse, topk, tok_local_rows): the merged output (identical on every rank), the global selection
    and this rank's rows of it."""
    dev = q.device
    world, rank = shard.world, shard.rank
    n_vis = max(0, min(shard.length, q_pos - shard.pad + 1)) // KPOOL
    n_loc = local_pool_count(n_vis, rank, world)
    ld_local = shard.pooled.shape[1]
    i32 = lambda v: torch.tensor(v, dtype=torch.int32, device=dev)  # noqa: E731
    # 1. local scores and selection over a pseudo-sequence of the rank's n_loc visible pools
    scores = torch.empty(1, ld_local, dtype=torch.float32, device=dev)
    topk_loc = torch.empty(1, select_k, dtype=torch.int32, device=dev)
    ws = torch.empty(glm_dsa_workspace_size(dims, GLM_OP_INDEX_SCORES_TOPK, 1, ld_local, select_k), dtype=torch.uint8,
                     device=dev)
    glm_index_scores_topk(dims, q_idx, w, shard.pooled, i32([0]), i32([KPOOL * n_loc - 1]), i32([0]),
                          i32([KPOOL * n_loc]), select_k, topk_loc, scores=scores, workspace=ws, stream=stream)
    cand_s = torch.empty(1, select_k, dtype=torch.float32, device=dev)
    cand_i = torch.empty(1, select_k, dtype=torch.int32, device=dev)
    glm_cp_candidates(scores, topk_loc, rank, world, cand_s, cand_i, stream=stream)
    # 2. the global selection (the same on every rank)
    all_s, all_i = all_gather(cand_s), all_gather(cand_i)          # [world, 1, select_k]
    topk = torch.empty(1, select_k, dtype=torch.int32, device=dev)
    n_sel = torch.empty(1, dtype=torch.int32, device=dev)
    glm_merge_topk(all_s, all_i, select_k, topk, n_sel=n_sel, stream=stream)
    # 3. its expansion through this rank's slot map: tokens held elsewhere map to -1
    rows = torch.empty(1, out_width, dtype=torch.int32, device=dev)
    glm_expand_selection(dims, topk, i32([0]), i32([q_pos]), i32([shard.pad]), i32([shard.length]), out_width,
                         n_sel=n_sel, slot_map=shard.slot_map, rows=rows, stream=stream)
    # 4. attention over this rank's rows, then the log-sum-exp merge of every rank's part
    H = q.shape[1]
    out_part = torch.empty(1, H, 512, dtype=torch.bfloat16, device=dev)
    o32_part = torch.empty(1, H, 512, dtype=torch.float32, device=dev)
    lse_part = torch.empty(1, H, dtype=torch.float32, device=dev)
    ws_m = torch.empty(glm_dsa_workspace_size(dims, GLM_OP_SPARSE_MLA, 1, width=out_width), dtype=torch.uint8,
                       device=dev)
    glm_sparse_mla_decode(dims, q, shard.cache, rows, sm_scale, out_part, ws_m, lse=lse_part, out_f32=o32_part,
                          stream=stream)
    all_o, all_l = all_gather(o32_part), all_gather(lse_part)      # [world, 1, H, 512], [world, 1, H]
    out = torch.empty(1, H, 512, dtype=torch.bfloat16, device=dev)
    out_f32 = torch.empty(1, H, 512, dtype=torch.float32, device=dev)
    lse = torch.empty(1, H, dtype=torch.float32, device=dev)
    glm_lse_merge(dims, all_o, all_l, out, out_f32=out_f32, lse=lse, stream=stream)
    return out, out_f32, lse, topk, rows


def torch_all_gather(group=None):
    """all_gather for cp_decode over a torch.distributed group (rank order)."""
    import torch.distributed as dist

    def gather(t):
        world = dist.get_world_size(group)
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out
    return gather
