"""GPU parity of the INT8 indexer state ("GLM-5.3-Flash" pypto-lib page, 'What is quantized': the
indexer cache in INT8 with one FP32 scale per row) against the oracle.

* glm_kpool_build_q8 must equal the oracle's quantisation of the fp32 pools the same inputs give
  through glm_kpool_build, bit for bit (both quantise identical fp32 values with one recipe).
* The scores on the INT8 state must match the oracle's scores on the same codes and scales within
  the index-score tolerance; the selection and expansion must be exact on the kernel's own scores.
* The one-call step on the INT8 state must reproduce the separate calls exactly, and the whole
  long-decode step must agree with the oracle's step on the INT8 state.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from kpool_indexer_int8_b200 import pipeline as P
from synth import device as sdev
from tests.test_gpu_parity import (_selection_agrees, assert_attention_close, assert_bf16_is_rounded_f32, np_,
                                   score_rel_err)

pytestmark = pytest.mark.gpu

CASES = [synth.TINY_DECODE, synth.PADDING_DECODE,
         synth.custom("q8_multi", (0, 3, 0, 1), (9000, 4099, 20000, 33), n_heads=64, select_k=512,
                      out_width=2176, permute_slots=True, seed=41)]


def _pairs(inp, cuda, **kw):
    """The same inputs loaded twice: fp32 pooled keys and the INT8 state."""
    bf = sdev.allocate_for(inp, cuda, **kw)
    sdev.load(inp, bf, build_prefix=True)
    bq = sdev.allocate_for(inp, cuda, q8=True, **kw)
    sdev.load(inp, bq, build_prefix=True)
    return bf, bq


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_kpool_q8_is_the_quantised_fp32_pool(cuda, wl):
    inp = synth.generate(wl)
    bf, bq = _pairs(inp, cuda)
    P.build_pools(bf)
    P.build_pools(bq)          # the step's new pools too
    torch.cuda.synchronize()
    pf = np_(bf.pooled)
    codes, scales = np_(bq.pooled_codes), np_(bq.pooled_scales)
    for s in range(wl.batch):
        n = min(int(inp.len[s]) // 4, pf.shape[1])
        want_c, want_s = oracle.pool_q8(pf[s, :n])
        assert np.array_equal(codes[s, :n], want_c), s
        assert np.array_equal(scales[s, :n], want_s), s


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_index_q8_scores_and_exact_selection(cuda, wl):
    inp = synth.generate(wl)
    b = sdev.allocate_for(inp, cuda, keep_scores=True, q8=True)
    sdev.load(inp, b, build_prefix=True)
    for t in (b.topk, b.n_sel, b.tok, b.rows):
        t.fill_(4242)
    b.ws_index.fill_(0xA5)
    b.ws_index[-256:].zero_()
    P.index_topk_expand(b)
    torch.cuda.synchronize()
    assert int(b.ws_index[-256:-252].view(torch.int32).item()) == 0
    codes, scales = np_(b.pooled_codes), np_(b.pooled_scales)
    sg, tg, ng, tokg, rowg = np_(b.scores), np_(b.topk), np_(b.n_sel), np_(b.tok), np_(b.rows)
    for n in range(len(inp.q_pos)):
        s = int(inp.q_seq[n])
        nv = oracle.n_visible_pools(inp.pad[s], inp.len[s], inp.q_pos[n])
        so = oracle.index_scores_q8(inp.q_idx[n], inp.w[n], codes[s], scales[s], nv)
        assert score_rel_err(sg[n, :nv], so) <= 1e-4, n
        want, n_sel = oracle.topk_pools(sg[n, :nv].astype(np.float64), wl.select_k)
        assert ng[n] == n_sel and np.array_equal(tg[n], want), n
        want_tok, _ = oracle.expand_selection(want, n_sel, inp.pad[s], inp.len[s], inp.q_pos[n], wl.out_width)
        assert np.array_equal(tokg[n], want_tok), n
        sm = inp.slot_map[s]
        assert np.array_equal(rowg[n], np.where(want_tok >= 0, sm[np.maximum(want_tok, 0)], -1)), n


def test_q8_step_equals_separate_calls(cuda):
    inp = synth.generate(CASES[2])
    outs = []
    for runner in (P.run_stages, P.run_step):
        b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True, q8=True)
        sdev.load(inp, b, build_prefix=True)
        runner(b)
        torch.cuda.synchronize()
        outs.append(b)
    a, c = outs
    for name in ("cache", "pooled_codes", "pooled_scales", "scores", "topk", "n_sel", "tok", "rows", "out_f32", "lse"):
        assert torch.equal(getattr(a, name), getattr(c, name)), name


def test_q8_long_decode_step_matches_oracle(cuda):
    # the benchmark workload on the INT8 state: the oracle selects on its own scores of the same
    # codes and scales; the GPU's pools may differ from it only inside the 1e-4 tie band
    inp = synth.generate(synth.LONG_DECODE)
    b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True, q8=True)
    sdev.load(inp, b, build_prefix=True)
    P.run_step(b)
    torch.cuda.synchronize()
    cache_o = oracle.build_cache(inp)
    assert np.array_equal(np_(b.cache[-4096:]), cache_o[-4096:])
    codes, scales = np_(b.pooled_codes), np_(b.pooled_scales)
    n = 0
    s = int(inp.q_seq[n])
    nv = oracle.n_visible_pools(inp.pad[s], inp.len[s], inp.q_pos[n])
    so = oracle.index_scores_q8(inp.q_idx[n], inp.w[n], codes[s], scales[s], nv)
    sg = np_(b.scores)
    assert score_rel_err(sg[n, :nv], so) <= 1e-4
    pools_o = oracle.build_pools(inp)
    r = oracle.decode_query(inp, n, cache_o, pools_o, scores_override=so)
    assert np_(b.n_sel)[n] == r["n_sel"]
    assert _selection_agrees(np_(b.topk)[n], r["topk"], so, r["n_sel"]) == 0
    assert np.array_equal(np_(b.tok)[n], r["tok"]) and np.array_equal(np_(b.rows)[n], r["rows"])
    assert_attention_close(np_(b.out_f32)[n], r["out"], "q8 long decode")
    assert_bf16_is_rounded_f32(np_(b.out[n].view(torch.int16)).view(np.uint16), np_(b.out_f32)[n])
