"""Context-parallel decode (kpool_indexer_int8_b200.cp) on one GPU, its ranks emulated.

Each emulated rank runs cp_decode on its own share of one sequence (its pools at local indices, the
cache rows of its tokens, a slot map to them) in a thread of its own; the all-gathers are host-side
stand-ins that stack every rank's tensor in rank order once all have arrived. No kernel of one rank
ever waits for another's (the exchange is on the host), so the ranks' kernels may run in any order.
Every rank must produce the single-GPU selection of the oracle and its attention within the
attention tolerance, and the ranks' merged outputs must be bit-identical."""
import threading

import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth
from kpool_indexer_int8_b200 import cp
from kpool_indexer_int8_b200 import pipeline as P
from synth import device as sdev

pytestmark = pytest.mark.gpu


class _HostGather:
    def __init__(self, world):
        self.world, self.items, self.barrier, self.lock = world, {}, threading.Barrier(world), threading.Lock()
        self.round = [0] * world

    def fn(self, rank):
        def gather(t):
            k = self.round[rank]
            self.round[rank] += 1
            torch.cuda.synchronize()
            with self.lock:
                self.items[(k, rank)] = t.clone()
            self.barrier.wait()
            out = torch.stack([self.items[(k, r)] for r in range(self.world)])
            self.barrier.wait()
            return out
        return gather


@pytest.mark.parametrize("world", [2, 3, 4])
def test_context_parallel_decode_matches_the_oracle(cuda, world):
    wl = synth.custom("cp_gpu", (5,), (16387,), n_heads=16, select_k=128, out_width=515, seed=31)
    inp = synth.generate(wl)
    b = sdev.allocate_for(inp, cuda)
    sdev.load(inp, b, build_prefix=True)
    P.run_step(b)                         # store the query token's row and build its pool
    torch.cuda.synchronize()
    pad, length, qp = int(inp.pad[0]), int(inp.len[0]), int(inp.q_pos[0])
    n_pools = length // 4
    ld_tokens = b.k.shape[1]
    shards = []
    for r in range(world):
        own_pools = torch.arange(r, n_pools, world, device=cuda)
        ld_local = max(1, (b.pooled.shape[1] + world - 1) // world)
        pooled = torch.zeros(1, ld_local, 128, dtype=torch.float32, device=cuda)
        pooled[0, :own_pools.numel()] = b.pooled[0, own_pools]
        toks = [t for t in range(pad, pad + length) if cp.owns_token(pad, length, t, r, world)]
        rows_g = b.slot_map[0, toks]                              # the global cache rows of its tokens
        cache = b.cache[rows_g].clone()
        slot_map = torch.full((1, ld_tokens), -1, dtype=torch.int64, device=cuda)
        slot_map[0, toks] = torch.arange(len(toks), device=cuda)
        shards.append(cp.CpShard(r, world, pooled, cache, slot_map, pad, length))
    g = _HostGather(world)
    res = [None] * world

    def run(r):
        res[r] = cp.cp_decode(b.dims, shards[r], b.q_idx, b.w, b.q, qp, wl.select_k, wl.out_width, inp.sm_scale,
                              g.fn(r))
        torch.cuda.synchronize()

    th = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=300)
    assert all(x is not None for x in res)
    # the ranks' merged selection is the one-GPU step's (the same per-pool score arithmetic), and the
    # attention over it is the oracle's over the same rows
    cache_o = oracle.build_cache(inp)
    want_topk = b.topk[0].cpu().numpy()
    tok, _ = oracle.expand_selection(want_topk, int(b.n_sel[0].item()), pad, length, qp, wl.out_width)
    rows_all = oracle.rows_from_tokens(tok, inp.slot_map[0])
    ref_out, ref_lse = oracle.sparse_mla(inp.q[0], cache_o, rows_all, inp.sm_scale)
    for r in range(world):
        out, out_f32, lse, topk, rows = res[r]
        assert np.array_equal(topk[0].cpu().numpy(), want_topk), r
        g32 = out_f32[0].cpu().numpy().astype(np.float64)
        err = np.abs(g32 - ref_out).max()
        rel = np.linalg.norm(g32 - ref_out) / np.linalg.norm(ref_out)
        assert err <= 1e-2 and rel <= 5e-3, (r, err, rel)
        np.testing.assert_allclose(lse[0].cpu().numpy(), ref_lse, atol=1e-3, rtol=0)
        assert torch.equal(out_f32, res[0][1]) and torch.equal(lse, res[0][2])
    # every selected token is attended by exactly one rank
    held = sum(int((res[r][4] >= 0).sum()) for r in range(world))
    assert held == int((tok >= 0).sum())
