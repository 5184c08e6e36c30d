"""Pins of the oracle's context-parallel merges against their definitions' consequences: the merge
of an interleaved split's local selections is the selection over all pools (brute force by
Python's sort, ties to the lower id), and the log-sum-exp merge of attention over a split of the
rows is the attention over all rows; plus the bookkeeping of which rank holds which pool."""
import numpy as np
import pytest

import oracle
import synth


@pytest.mark.parametrize("world,n,S", [(2, 300, 16), (3, 1000, 64), (8, 4096, 512), (4, 10, 16)])
def test_merge_of_local_selections_is_the_global_selection(world, n, S):
    rng = np.random.default_rng(world * n)
    scores = np.round(rng.standard_normal(n) * 4) / 4          # heavy ties: the id rule decides
    scores[rng.random(n) < 0.05] = -0.0
    cand_s, cand_i = [], []
    for r in range(world):
        own = np.arange(r, n, world)
        loc, cnt = oracle.topk_pools(scores[own], S)             # local indices
        cand_s.append(np.where(loc >= 0, scores[own][np.maximum(loc, 0)], 0.0))
        cand_i.append(np.where(loc >= 0, own[np.maximum(loc, 0)], -1))
    got, cnt = oracle.merge_topk(np.concatenate(cand_s), np.concatenate(cand_i), S)
    want = sorted(range(n), key=lambda p: (-(scores[p] + 0.0), p))[:S]
    assert cnt == min(S, n)
    assert list(got[:cnt]) == want and (got[cnt:] == -1).all()


def test_lse_merge_of_a_row_split_is_the_attention_over_all_rows():
    rng = np.random.default_rng(4)
    n_rows, H = 600, 16
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    cache = np.zeros((n_rows, 528), np.int8)
    oracle.store_int8(lat, np.arange(n_rows, dtype=np.int64), cache)
    q = synth.f32_to_bf16_bits(rng.standard_normal((H, 512)).astype(np.float32))
    rows = rng.choice(n_rows, size=300, replace=False).astype(np.int32)
    sm = 512 ** -0.5
    full, lse_full = oracle.sparse_mla(q, cache, rows, sm)
    for world in (2, 3, 5):
        parts = [oracle.sparse_mla(q, cache, np.where(np.arange(300) % world == r, rows, -1), sm)
                 for r in range(world)]
        out, lse = oracle.lse_merge([p[0] for p in parts], [p[1] for p in parts])
        np.testing.assert_allclose(out, full, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_full, rtol=0, atol=1e-12)
    # an empty part (no rows: out 0, lse -inf) changes nothing; one part returns itself
    e_out, e_lse = oracle.sparse_mla(q, cache, np.full(300, -1, np.int32), sm)
    out, lse = oracle.lse_merge([full, e_out], [lse_full, e_lse])
    np.testing.assert_allclose(out, full, atol=1e-15)
    out, lse = oracle.lse_merge([full], [lse_full])
    np.testing.assert_allclose(out, full, atol=0)
    # two parts with equal lse: the plain mean
    a, b = rng.standard_normal((2, H, 512))
    out, lse = oracle.lse_merge([a, b], [np.full(H, 1.5), np.full(H, 1.5)])
    np.testing.assert_allclose(out, (a + b) / 2, atol=1e-15)
    np.testing.assert_allclose(lse, 1.5 + np.log(2), atol=1e-15)
