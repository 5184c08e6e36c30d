"""GPU parity of the many-query scoring path ("Module glm5next_dsa_ref": index_scores, the relu
head-weighted sum; a prefill chunk's queries scored together, pooled keys on the MMA M dimension)
against the oracle, through glm_index_scores_topk / glm_index_topk_expand with at least 128 queries.

* every score of a visible pool within the index-score tolerance (|g - o| / max(|o|, 1e-3 max|o|)
  <= 1e-4) of the oracle's fp64 score on the same fp32 pooled keys; -inf past the visible pools; a
  query of no valid sequence gets an all -inf row and an empty selection (-1 everywhere);
* n_sel exact; the selection equal to the oracle's top-k on its scores up to exchanges within the
  tie band (1e-4 of the select_k-th score); the expansion of the GPU's own selection bit-exact;
* shapes that reach every branch: queries of three sequences interleaved (groups mixing
  sequences), a padded last group, a ragged last tile (pools not a multiple of 256 nor of 128), a
  sequence that sees no pool of most tiles, zero and tiny pooled keys, keys whose magnitude varies
  by orders between pools.
"""
import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth
from tests.test_gpu_parity import _selection_agrees, np_, score_rel_err, to_dev

pytestmark = pytest.mark.gpu


def _case(seed, n_q, pads, lens, ld):
    rng = np.random.default_rng(seed)
    B = len(pads)
    mag = np.exp(2.0 * rng.standard_normal((B, ld, 1)))
    pooled = (rng.standard_normal((B, ld, 128)) * mag).astype(np.float32)
    pooled[0, 3] = 0.0
    pooled[B - 1, 5] *= np.float32(1e-30)
    q = synth.f32_to_bf16_bits(rng.standard_normal((n_q, 32, 128)).astype(np.float32))
    w = rng.random((n_q, 32)).astype(np.float32)
    q_seq = rng.integers(0, B, n_q).astype(np.int32)
    q_pos = np.array([rng.integers(pads[s], pads[s] + lens[s]) for s in q_seq], np.int32)
    q_pos[:B] = [pads[s] + lens[s] - 1 for s in range(B)]         # the last position of each sequence
    q_seq[n_q // 2] = B + 3                                       # no valid sequence
    return pooled, q, w, q_seq, q_pos, np.array(pads, np.int32), np.array(lens, np.int32)


def _oracle_rows(pooled, q, w, q_seq, q_pos, pad, length):
    res = []
    for n in range(len(q_seq)):
        s = int(q_seq[n])
        if s < 0 or s >= len(pad):
            res.append(np.empty(0))
            continue
        nv = oracle.n_visible_pools(pad[s], length[s], q_pos[n])
        res.append(oracle.index_scores(q[n], w[n], pooled[s], nv))
    return res


CASES = [
    # n_q, pads, lens, ld: 301 queries (a padded last group), 700 pools (the last tile 188 rows: a
    # full half and 60 rows), a short sequence (22 pools: nothing visible in tiles 1 and 2)
    (301, (0, 3, 6), (2800, 1601, 90), 700),
    # one sequence, 128 queries (the smallest many-query count), 1,030 pools
    (128, (0,), (4120,), 1030),
]


@pytest.mark.parametrize("n_q,pads,lens,ld", CASES)
@pytest.mark.parametrize("select_k", [64, 512])
def test_many_query_scores_and_selection(cuda, n_q, pads, lens, ld, select_k):
    pooled, q, w, q_seq, q_pos, pad, length = _case(n_q + select_k, n_q, pads, lens, ld)
    dims = kp.make_dims(16)
    scores = torch.full((n_q, ld), 12345.0, dtype=torch.float32, device=cuda)
    topk = torch.full((n_q, select_k), 555, dtype=torch.int32, device=cuda)
    n_sel = torch.full((n_q,), 777, dtype=torch.int32, device=cuda)
    ws = torch.full((kp.glm_dsa_workspace_size(dims, kp.GLM_OP_INDEX_SCORES_TOPK, n_q, ld, select_k),),
                    0xA5, dtype=torch.uint8, device=cuda)
    status = ws[-256:-252].view(torch.int32)
    status.zero_()
    kp.glm_index_scores_topk(dims, to_dev(q, torch.bfloat16, cuda), to_dev(w, torch.float32, cuda),
                             to_dev(pooled, torch.float32, cuda), to_dev(q_seq, torch.int32, cuda),
                             to_dev(q_pos, torch.int32, cuda), to_dev(pad, torch.int32, cuda),
                             to_dev(length, torch.int32, cuda), select_k, topk, n_sel=n_sel, scores=scores,
                             workspace=ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    sg, tg, ng = np_(scores), np_(topk), np_(n_sel)
    diffs = 0
    for n, so in enumerate(_oracle_rows(pooled, q, w, q_seq, q_pos, pad, length)):
        nv = len(so)
        assert score_rel_err(sg[n, :nv], so) <= 1e-4, n
        assert np.isneginf(sg[n, nv:]).all(), n
        want, k = oracle.topk_pools(so, select_k)
        assert ng[n] == k, n
        diffs += _selection_agrees(tg[n], want, so, k)
    assert diffs <= n_q // 20


def test_many_query_expansion(cuda):
    n_q, pads, lens, ld, S, W = 200, (0, 5), (3000, 1200), 750, 64, 4 * 64 + 3
    pooled, q, w, q_seq, q_pos, pad, length = _case(7, n_q, pads, lens, ld)
    dims = kp.make_dims(16)
    topk = torch.full((n_q, S), 555, dtype=torch.int32, device=cuda)
    n_sel = torch.full((n_q,), 777, dtype=torch.int32, device=cuda)
    tok = torch.full((n_q, W), 4242, dtype=torch.int32, device=cuda)
    ws = torch.full((kp.glm_dsa_workspace_size(dims, kp.GLM_OP_INDEX_SCORES_TOPK, n_q, ld, S),), 0xA5,
                    dtype=torch.uint8, device=cuda)
    kp.glm_index_topk_expand(dims, to_dev(q, torch.bfloat16, cuda), to_dev(w, torch.float32, cuda),
                             to_dev(pooled, torch.float32, cuda), to_dev(q_seq, torch.int32, cuda),
                             to_dev(q_pos, torch.int32, cuda), to_dev(pad, torch.int32, cuda),
                             to_dev(length, torch.int32, cuda), S, topk, W, n_sel=n_sel, tok=tok, workspace=ws)
    torch.cuda.synchronize()
    tg, ng, tokg = np_(topk), np_(n_sel), np_(tok)
    for n in range(n_q):
        s = int(q_seq[n])
        if s < 0 or s >= len(pads):
            assert ng[n] == 0 and (tg[n] == -1).all() and (tokg[n] == -1).all(), n
            continue
        want_tok, _ = oracle.expand_selection(tg[n], ng[n], pad[s], length[s], q_pos[n], W)
        assert np.array_equal(tokg[n], want_tok), n
