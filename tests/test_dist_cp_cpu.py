"""Context-parallel decode on CPU with the gloo backend, world sizes 2 and 3.

Each rank holds the pools the bookkeeping of kpool_indexer_int8_b200.cp assigns it (p = r + world i,
with the tokens of those pools and the tail when it would own the next pool); the oracle stands in
for the kernels on each rank (local scores, local selection, attention over the rank's own rows),
and torch.distributed.all_gather carries the candidates and the attention parts between the
processes. Every rank must end with the single-process oracle's selection and attention."""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from kpool_indexer_int8_b200 import cp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))

    def all_gather(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t)
        return np.stack([p.numpy() for p in parts])

    wl = synth.custom("cp", (3,), (2003,), n_heads=16, select_k=64, out_width=259, seed=21)
    inp = synth.generate(wl)
    cache = oracle.build_cache(inp)
    pools = oracle.build_pools(inp)[0]
    pad, length, qp = int(inp.pad[0]), int(inp.len[0]), int(inp.q_pos[0])
    n_vis = oracle.n_visible_pools(pad, length, qp)
    S, W = wl.select_k, wl.out_width
    # this rank's pools (local index i = global pool r + world i) and their scores
    n_loc = cp.local_pool_count(n_vis, rank, world)
    own = np.arange(n_loc) * world + rank
    assert all(cp.pool_owner(int(p), world) == rank and cp.local_index(int(p), world) == i for i, p in enumerate(own))
    scores_loc = oracle.index_scores(inp.q_idx[0], inp.w[0], pools[own], n_loc)
    loc, cnt = oracle.topk_pools(scores_loc, S)
    cand_s = np.where(loc >= 0, scores_loc[np.maximum(loc, 0)], 0.0)
    cand_i = np.where(loc >= 0, loc * world + rank, -1)          # the glm_cp_candidates mapping
    topk, n_sel = oracle.merge_topk(all_gather(cand_s), all_gather(cand_i), S)
    tok, _ = oracle.expand_selection(topk, n_sel, pad, length, qp, W)
    rows = oracle.rows_from_tokens(tok, inp.slot_map[0])
    mine = np.array([t >= 0 and cp.owns_token(pad, length, int(t), rank, world) for t in tok])
    out_p, lse_p = oracle.sparse_mla(inp.q[0], cache, np.where(mine, rows, -1), inp.sm_scale)
    out, lse = oracle.lse_merge(all_gather(out_p), all_gather(lse_p))
    ref = oracle.decode_query(inp, 0, cache, oracle.build_pools(inp))
    res = {"rank": rank, "topk_equal": bool(np.array_equal(topk, ref["topk"])),
           "n_sel": int(n_sel), "ref_n_sel": int(ref["n_sel"]),
           "tok_equal": bool(np.array_equal(tok, ref["tok"])),
           "out_err": float(np.abs(out - ref["out"]).max()), "lse_err": float(np.abs(lse - ref["lse"]).max()),
           "own_rows": int(mine.sum()), "all_rows": int((tok >= 0).sum()), "out0": out[0, :4].tolist()}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_matches_single_process(tmp_path, world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    for r in res:
        assert r["topk_equal"] and r["tok_equal"] and r["n_sel"] == r["ref_n_sel"]
        assert r["out_err"] <= 1e-12 and r["lse_err"] <= 1e-12
        assert r["out0"] == res[0]["out0"]                      # identical on every rank
    assert sum(r["own_rows"] for r in res) == res[0]["all_rows"]   # every selected row held once
