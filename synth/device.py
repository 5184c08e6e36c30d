"""Upload a synthetic workload state into the CUDA path's device buffers.

Copies only: the arrays drawn by ``synth.generate`` go to the GPU as they are. The prefix (every
token before the query positions) is then written into the int8 cache and pooled into the
indexer state by the library's own entry points -- the set-up a model would have done on earlier
steps -- while the query positions' tokens are left as the step's inputs.
"""
from __future__ import annotations

import numpy as np
import torch

from kpool_indexer_int8_b200 import pipeline as P

from . import Inputs


def _t(a, dtype, device):
    if dtype == torch.bfloat16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


def step_split(inp: Inputs):
    """(prefix lengths per sequence, packed indices of the step's new tokens)."""
    new = inp.new_token_mask()
    n_new_seq = np.zeros(inp.wl.batch, dtype=np.int64)
    for qs in inp.q_seq:
        n_new_seq[qs] += 1
    return (inp.len - n_new_seq).astype(np.int32), np.nonzero(new)[0]


def allocate_for(inp: Inputs, device, keep_scores=False, keep_f32=False, q8=False, fp8=False,
                 fp4=False) -> P.DecodeBuffers:
    prefix, new_idx = step_split(inp)
    per_seq_new = int(max(1, (inp.len - prefix).max()))
    max_new_pools = per_seq_new // P.KPOOL + 1
    return P.allocate(inp.wl.n_heads, inp.wl.batch, inp.ld_tokens, inp.n_rows, len(inp.q_pos),
                      len(new_idx), inp.wl.select_k, inp.wl.out_width, inp.sm_scale,
                      inp.wl.ln_eps, max_new_pools, device, keep_scores=keep_scores,
                      keep_f32=keep_f32, q8=q8, fp8=fp8, fp4=fp4)


def load(inp: Inputs, b: P.DecodeBuffers, build_prefix: bool = True) -> None:
    """Copy the state and the step inputs of ``inp`` into ``b``; store and pool the prefix."""
    dev = b.cache.device
    prefix, new_idx = step_split(inp)
    b.k.copy_(_t(inp.k, torch.bfloat16, dev))
    b.gate.copy_(_t(inp.gate, torch.bfloat16, dev))
    b.ln_w.copy_(_t(inp.ln_w, torch.float32, dev))
    b.ln_b.copy_(_t(inp.ln_b, torch.float32, dev))
    b.pad.copy_(_t(inp.pad, torch.int32, dev))
    b.len.copy_(_t(inp.len, torch.int32, dev))
    b.slot_map.copy_(_t(inp.slot_map, torch.int64, dev))
    b.q_idx.copy_(_t(inp.q_idx, torch.bfloat16, dev))
    b.w.copy_(_t(inp.w, torch.float32, dev))
    b.q.copy_(_t(inp.q, torch.bfloat16, dev))
    b.q_seq.copy_(_t(inp.q_seq, torch.int32, dev))
    b.q_pos.copy_(_t(inp.q_pos, torch.int32, dev))
    b.new_latent.copy_(_t(inp.latent[new_idx], torch.bfloat16, dev))
    b.new_slots.copy_(_t(inp.slots[new_idx], torch.int64, dev))
    b.pool_begin.copy_(_t(prefix // P.KPOOL, torch.int32, dev))
    if build_prefix:
        keep = np.ones(inp.latent.shape[0], dtype=bool)
        keep[new_idx] = False
        idx = np.nonzero(keep)[0]
        step = 1 << 18
        for s in range(0, len(idx), step):
            sl = idx[s:s + step]
            lat = _t(inp.latent[sl], torch.bfloat16, dev)
            slots = _t(inp.slots[sl], torch.int64, dev)
            from kpool_indexer_int8_b200 import glm_kv_store_fp4, glm_kv_store_fp8, glm_kv_store_int8
            store = glm_kv_store_fp4 if b.fp4 else glm_kv_store_fp8 if b.fp8 else glm_kv_store_int8
            store(b.dims, lat, slots, b.cache)
            del lat, slots
        plen = _t(prefix, torch.int32, dev)
        P.build_pools(b, length=plen, pool_begin=torch.zeros_like(b.pool_begin),
                      max_new_pools=b.pooled.shape[1])
    torch.cuda.synchronize(dev)
