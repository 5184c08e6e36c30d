"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the same seeded inputs.

Agreement rules
  * int8 cache rows, index lists (top-k ids, tokens, cache rows): bit-exact.
  * top-k: bit-exact when fed the oracle's scores rounded to fp32 (both sides select on the same
    fp32 values); in the chained path the GPU selection may differ from the oracle's only among
    pools whose oracle score lies within 1e-4 (relative) of the select_k-th score.
  * index scores: max over (n, p) of |g - o| / max(|o|, 1e-3 * max_p |o[n, p]|) <= 1e-4.
  * attention output: the fp32 output within max abs err <= 1e-2 and relative L2 error <= 5e-3
    of the oracle on the same int8 rows; the bf16 output equal to the fp32 output rounded to
    nearest-even bf16 (bit-exact: a bf16 value near 16 alone carries a 0.0625 rounding step, so
    the absolute bound is stated on the fp32 result); lse within 1e-3 absolute.
  * pooled keys (fp32 kernel, fp64 oracle): |g - o| <= 2e-5 * (1 + |o|). Derivation: the LayerNorm
    sums 128 fp32 terms (relative error <= ~128 * 2**-24 = 7.6e-6 of the largest term, typically
    ~1e-6), the slot softmax adds a few ulps, so 2e-5 leaves a margin of ~3x over the worst case.
"""
import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth
from kpool_indexer_int8_b200 import pipeline as P
from synth import device as sdev

pytestmark = pytest.mark.gpu

POISON = 0x5A


def np_(t):
    return t.detach().cpu().numpy()


def to_dev(a, dtype, dev):
    return sdev._t(a, dtype, dev)


def score_rel_err(g, o):
    o = np.asarray(o, np.float64)
    g = np.asarray(g, np.float64)
    if o.size == 0:
        return 0.0
    den = np.maximum(np.abs(o), 1e-3 * np.abs(o).max())
    den[den == 0] = 1.0
    return float((np.abs(g - o) / den).max())


def attn_errors(g, o):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    max_abs = float(np.abs(g - o).max()) if o.size else 0.0
    nrm = np.linalg.norm(o)
    rel_l2 = float(np.linalg.norm(g - o) / nrm) if nrm > 0 else float(np.linalg.norm(g))
    return max_abs, rel_l2


def assert_attention_close(g, o, what=""):
    max_abs, rel_l2 = attn_errors(g, o)
    assert max_abs <= 1e-2 and rel_l2 <= 5e-3, (what, max_abs, rel_l2)


def assert_bf16_is_rounded_f32(out_bf16_bits, out_f32):
    assert np.array_equal(np.asarray(out_bf16_bits, np.uint16),
                          synth.f32_to_bf16_bits(np.asarray(out_f32, np.float32)))


# ------------------------------------------------------------------------------------------------
# store_int8
# ------------------------------------------------------------------------------------------------

def _store_both(cuda, latent, slots, n_rows):
    dims = kp.make_dims(16)
    co = np.full((n_rows, 528), POISON, dtype=np.int8)
    ok = (slots >= 0) & (slots < n_rows)
    oracle.store_int8(latent[ok], slots[ok], co)
    cg = torch.full((n_rows, 528), POISON, dtype=torch.int8, device=cuda)
    kp.glm_kv_store_int8(dims, to_dev(latent, torch.bfloat16, cuda), to_dev(slots, torch.int64, cuda), cg)
    torch.cuda.synchronize()
    return np_(cg), co


@pytest.mark.parametrize("wl", [synth.TINY_DECODE, synth.PADDING_DECODE,
                                synth.custom("permuted", (0, 3), (1000, 517), permute_slots=True,
                                             outlier_frac=0.05)])
def test_store_int8_bit_exact(cuda, wl):
    inp = synth.generate(wl)
    g, o = _store_both(cuda, inp.latent, inp.slots, inp.n_rows)
    assert np.array_equal(g, o)


def test_store_int8_edge_rows(cuda):
    # zero rows (amax floor), exact halves (ties to even), the largest bf16 magnitudes, tiny values,
    # negative slots (no write) and slots past the cache (skipped, never written)
    rng = np.random.default_rng(0)
    x = np.zeros((8, 512), np.float32)
    x[1, :11] = [127, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -0.5, 126.5, -127, -1.5]
    x[2] = rng.standard_normal(512) * 1e-7
    x[3] = rng.standard_normal(512) * 3e38 / 5
    x[4] = -np.abs(rng.standard_normal(512))
    x[5, 0] = 1.0
    x[6] = rng.standard_normal(512)
    x[7] = rng.standard_normal(512)
    lat = synth.f32_to_bf16_bits(x)
    slots = np.array([0, 1, 2, 3, 4, -1, 6, 9], dtype=np.int64)   # 9 >= n_rows: skipped
    g, o = _store_both(cuda, lat, slots, 8)
    assert np.array_equal(g, o)
    assert (g[5] == POISON).all() and (g[7] == POISON).all()
    assert list(g[1, :11]) == [127, 2, 4, -2, -4, 0, 2, 0, 126, -127, -2]


def test_store_int8_full_size(cuda):
    # the long-decode cache: 262,144 rows with 1% outliers, compared in full
    inp = synth.generate(synth.LONG_DECODE)
    g, o = _store_both(cuda, inp.latent, inp.slots, inp.n_rows)
    assert np.array_equal(g, o)


# ------------------------------------------------------------------------------------------------
# kpool_build
# ------------------------------------------------------------------------------------------------

def _pooled_close(g, o):
    assert g.shape == o.shape
    err = np.abs(g.astype(np.float64) - o)
    assert (err <= 2e-5 * (1 + np.abs(o))).all(), float((err / (1 + np.abs(o))).max())


@pytest.mark.parametrize("wl", [synth.TINY_DECODE, synth.PADDING_DECODE])
def test_kpool_build_full_and_incremental(cuda, wl):
    inp = synth.generate(wl)
    pools_o = oracle.build_pools(inp)
    b = sdev.allocate_for(inp, cuda)
    sdev.load(inp, b, build_prefix=False)
    b.pooled.fill_(float("nan"))
    n_pools = torch.full((wl.batch,), -7, dtype=torch.int32, device=cuda)
    kp.glm_kpool_build(b.dims, b.k, b.gate, b.ln_w, b.ln_b, wl.ln_eps, b.pad, b.len, b.pooled,
                       pool_begin=None, max_new_pools=b.pooled.shape[1], n_pools=n_pools)
    pg = np_(b.pooled)
    assert list(np_(n_pools)) == [p.shape[0] for p in pools_o]
    for s, po in enumerate(pools_o):
        _pooled_close(pg[s, :po.shape[0]], po)
        assert np.isnan(pg[s, po.shape[0]:]).all()        # no pool past the last complete one
    # incremental: rebuild only pools [n-3, n-1) of each sequence into a fresh buffer
    b.pooled.fill_(float("nan"))
    nps = np.array([p.shape[0] for p in pools_o])
    begin = np.maximum(nps - 3, 0).astype(np.int32)
    kp.glm_kpool_build(b.dims, b.k, b.gate, b.ln_w, b.ln_b, wl.ln_eps, b.pad, b.len, b.pooled,
                       pool_begin=to_dev(begin, torch.int32, cuda), max_new_pools=2)
    pg = np_(b.pooled)
    for s, po in enumerate(pools_o):
        lo, hi = begin[s], min(begin[s] + 2, po.shape[0])
        _pooled_close(pg[s, lo:hi], po[lo:hi])
        assert np.isnan(pg[s, :lo]).all() and np.isnan(pg[s, hi:]).all()


# ------------------------------------------------------------------------------------------------
# index scores and top-k
# ------------------------------------------------------------------------------------------------

def _oracle_scores_on(inp, pooled32):
    res = []
    for n in range(len(inp.q_pos)):
        s = int(inp.q_seq[n])
        nv = oracle.n_visible_pools(inp.pad[s], inp.len[s], inp.q_pos[n])
        res.append(oracle.index_scores(inp.q_idx[n], inp.w[n], pooled32[s], nv))
    return res


@pytest.mark.parametrize("wl", [synth.TINY_DECODE, synth.PADDING_DECODE,
                                synth.custom("causal", (0,), (3000,), select_k=64, chunk=37)])
def test_index_scores_match_oracle(cuda, wl):
    inp = synth.generate(wl)
    pools_o = oracle.build_pools(inp)
    b = sdev.allocate_for(inp, cuda, keep_scores=True)
    sdev.load(inp, b, build_prefix=False)
    ld = b.pooled.shape[1]
    p32 = np.zeros((wl.batch, ld, 128), np.float32)          # the oracle's pools rounded to fp32
    for s, po in enumerate(pools_o):
        p32[s, :po.shape[0]] = po
    b.pooled.copy_(torch.from_numpy(p32))
    b.scores.fill_(12345.0)
    P.index_topk(b)
    sg = np_(b.scores)
    for n, so in enumerate(_oracle_scores_on(inp, p32)):
        assert score_rel_err(sg[n, :len(so)], so) <= 1e-4
        assert np.isneginf(sg[n, len(so):]).all()


def _topk_given(cuda, scores32, n_vis, S):
    nq, ld = scores32.shape
    topk = torch.full((nq, S), 777, dtype=torch.int32, device=cuda)
    n_sel = torch.full((nq,), 777, dtype=torch.int32, device=cuda)
    dims = kp.make_dims(16)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_TOPK_POOLS, nq, ld, S), dtype=torch.uint8,
                     device=cuda)
    ws.fill_(0xA5)                                   # contents on entry must not matter
    kp.glm_topk_pools(torch.from_numpy(scores32).to(cuda), to_dev(n_vis, torch.int32, cuda), S, topk,
                      n_sel=n_sel, workspace=ws)
    return np_(topk), np_(n_sel)


@pytest.mark.parametrize("n,S,ties", [(0, 8, False), (5, 8, False), (8, 8, False), (300, 16, False),
                                      (300, 16, True), (5000, 512, True), (5000, 1, True),
                                      (4100, 2048, False), (65536, 512, False), (65536, 512, True),
                                      (100000, 2048, True), (65536, 512, "uniform"),
                                      (65536, 512, "equal"), (70000, 2048, "uniform")])
def test_topk_bit_exact_on_oracle_scores(cuda, n, S, ties):
    # "uniform" puts ~8000 scores in the boundary bin of the 11-bit histogram (the path that selects
    # from the global list); "equal" leaves only the pool ids to decide
    rng = np.random.default_rng(n + S)
    s = rng.standard_normal(max(n, 1)) * 20 + 60
    if ties == "uniform":
        s = rng.random(max(n, 1))
    elif ties == "equal":
        s = np.full(max(n, 1), 3.5)
    elif ties:
        s = np.round(s * 4) / 4                        # heavy ties
        s[rng.random(s.shape) < 0.05] = 0.0
        s[rng.random(s.shape) < 0.05] = -0.0
    s32 = s.astype(np.float32)
    scores = np.full((2, max(n, 1) + 3), np.nan, np.float32)   # entries past n_vis are never read
    scores[0, :max(n, 1)] = s32
    scores[1, :max(n, 1)] = -s32                        # negative scores too
    n_vis = np.array([n, max(0, n - 1)], dtype=np.int32)
    tg, ng = _topk_given(cuda, scores, n_vis, S)
    for q in range(2):
        want, n_sel = oracle.topk_pools(scores[q, :n_vis[q]].astype(np.float64), S)
        assert np.array_equal(tg[q], want), q
        assert ng[q] == n_sel


def test_index_topk_fused_selection(cuda):
    inp = synth.generate(synth.PADDING_DECODE)
    pools_o = oracle.build_pools(inp)
    b = sdev.allocate_for(inp, cuda)
    sdev.load(inp, b, build_prefix=False)
    p32 = np.zeros(tuple(b.pooled.shape), np.float32)
    for s, po in enumerate(pools_o):
        p32[s, :po.shape[0]] = po
    b.pooled.copy_(torch.from_numpy(p32))
    b.topk.fill_(555)
    P.index_topk(b)
    tg, ng = np_(b.topk), np_(b.n_sel)
    for n, so in enumerate(_oracle_scores_on(inp, p32)):
        want, n_sel = oracle.topk_pools(so, inp.wl.select_k)
        assert ng[n] == n_sel
        assert _selection_agrees(tg[n], want, so, n_sel) == 0


_FUSED_CASES = [synth.TINY_DECODE, synth.PADDING_DECODE,
                synth.custom("multi_q", (0, 3, 0, 1, 0, 2, 0, 0), (9000, 4099, 20000, 33, 64, 70001, 2048, 5),
                             n_heads=64, select_k=512, out_width=2176, permute_slots=True, seed=35),
                synth.custom("one_long", (1,), (131075,), n_heads=64, select_k=2048, out_width=8195, seed=36)]


@pytest.mark.parametrize("wl", _FUSED_CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("pattern", ["synth", "few", "equal", "signed", "wide", "lead", "trend"])
def test_fused_select_expand_bit_exact_on_own_scores(cuda, wl, pattern):
    # the one-launch scores + selection + expansion: its top-k rows must be exactly the oracle's
    # selection of the scores it wrote, and its tokens / rows exactly the oracle's expansion of
    # that selection ("few": 3 distinct pooled keys, "equal": one -- only pool ids decide;
    # "signed": head weights of both signs, so scores of both signs; "wide": signed, and pooled
    # keys scaled over 2^-60 .. 2^60, so a CTA's scores fill hundreds of 11-bit bins; "lead": the
    # first tile of every CTA's range scaled x8, so that the multi-CTA sample overstates the
    # scores and its threshold lets too few through; "trend": keys scaled up along the sequence,
    # so that the candidates crowd into the last CTAs' ranges)
    inp = synth.generate(wl)
    b = sdev.allocate_for(inp, cuda, keep_scores=True)
    sdev.load(inp, b, build_prefix=True)
    if pattern == "few":
        b.pooled.copy_(b.pooled[:, torch.arange(b.pooled.shape[1], device=cuda) % 3])
    elif pattern == "equal":
        b.pooled.copy_(b.pooled[:, :1].expand_as(b.pooled))
    if pattern in ("signed", "wide"):
        b.w.mul_(torch.where(torch.arange(b.w.shape[1], device=cuda) % 3 == 0, -1.5, 1.0))
    if pattern == "wide":
        e = (torch.arange(b.pooled.shape[1], device=cuda) * 37 % 121 - 60).float()
        b.pooled.mul_(torch.exp2(e)[None, :, None])
    if pattern in ("lead", "trend"):
        ld, n_q = b.pooled.shape[1], len(inp.q_pos)
        G = min(max(1, torch.cuda.get_device_properties(cuda).multi_processor_count // n_q), -(-ld // 64))
        p = torch.arange(ld, device=cuda)
        for n in range(n_q):
            s = int(inp.q_seq[n])
            nv = max(1, oracle.n_visible_pools(inp.pad[s], inp.len[s], inp.q_pos[n]))
            per = max(-(-nv // G), 64)
            f = torch.where(p % per < 64, 8.0, 1.0) if pattern == "lead" else 1.0 + 3.0 * p.float() / nv
            b.pooled[s].mul_(f[:, None])
    for t in (b.topk, b.n_sel, b.tok, b.rows):
        t.fill_(4242)
    b.scores.fill_(7.0)
    for _ in range(2):                      # twice: the multi-CTA words must be reset every call
        b.ws_index.fill_(0xA5)
        b.ws_index[-256:].zero_()           # the status word
        P.index_topk_expand(b)
    torch.cuda.synchronize()
    assert int(b.ws_index[-256:-252].view(torch.int32).item()) == 0
    sg, tg, ng, tokg, rowg = np_(b.scores), np_(b.topk), np_(b.n_sel), np_(b.tok), np_(b.rows)
    S, W = wl.select_k, wl.out_width
    for n in range(len(inp.q_pos)):
        s = int(inp.q_seq[n])
        nv = oracle.n_visible_pools(inp.pad[s], inp.len[s], inp.q_pos[n])
        assert np.isneginf(sg[n, nv:]).all()
        want, n_sel = oracle.topk_pools(sg[n, :nv].astype(np.float64), S)
        assert ng[n] == n_sel, n
        assert np.array_equal(tg[n], want), n
        want_tok, _ = oracle.expand_selection(want, n_sel, inp.pad[s], inp.len[s], inp.q_pos[n], W)
        assert np.array_equal(tokg[n], want_tok), n
        sm = inp.slot_map[s]
        assert np.array_equal(rowg[n], np.where(want_tok >= 0, sm[np.maximum(want_tok, 0)], -1)), n


def test_fused_entry_equals_separate_entries(cuda):
    inp = synth.generate(_FUSED_CASES[2])
    b = sdev.allocate_for(inp, cuda, keep_scores=True)
    sdev.load(inp, b, build_prefix=True)
    P.index_topk_expand(b)
    fused = [np_(t).copy() for t in (b.scores, b.topk, b.n_sel, b.tok, b.rows)]
    for t in (b.scores, b.topk, b.n_sel, b.tok, b.rows):
        t.fill_(99)
    P.index_topk(b)
    P.expand(b)
    sep = [np_(t) for t in (b.scores, b.topk, b.n_sel, b.tok, b.rows)]
    for f, g in zip(fused, sep):
        assert np.array_equal(f, g)


def _selection_agrees(got, want, scores, n_sel):
    """The GPU selection against the oracle's (scores = the oracle's fp64 scores). Equal as sets,
    except that pools whose score is within 1e-4 (relative) of the select_k-th score may be
    exchanged; and in an order that is non-increasing in oracle score up to that tolerance (pools
    closer than the fp32 rounding of their scores may come in either order). Returns the number
    of exchanged pools."""
    assert (got[n_sel:] == -1).all()
    if n_sel == 0:
        return 0
    thr = scores[want[n_sel - 1]]
    tol = 1e-4 * max(abs(thr), 1e-30)
    g = got[:n_sel]
    assert (g >= 0).all() and (g < len(scores)).all() and len(set(g.tolist())) == n_sel
    gs, ws = set(g.tolist()), set(want[:n_sel].tolist())
    for p in gs ^ ws:
        assert abs(scores[p] - thr) <= tol, (p, scores[p], thr)
    sg = scores[g]
    suffix_max = np.maximum.accumulate(sg[::-1])[::-1]
    band = 1e-4 * np.maximum(np.abs(sg), 1e-30)
    assert (sg[:-1] >= suffix_max[1:] - band[:-1]).all(), "order not descending within tolerance"
    return len(gs ^ ws) // 2


def _expanded_is_valid(tok, rows, topk, n_sel, want_tok, inp, n):
    """Expanded tokens of a selection that matches the oracle's as a set: every 4-token block is
    the pool of the same position of the GPU's own top-k list, ascending; the tail and the -1
    padding equal the oracle's exactly; rows are the slot map of the tokens."""
    s = int(inp.q_seq[n])
    pad = int(inp.pad[s])
    for i in range(n_sel):
        assert list(tok[4 * i:4 * i + 4]) == [pad + 4 * int(topk[i]) + j for j in range(4)]
    assert np.array_equal(tok[4 * n_sel:], want_tok[4 * n_sel:])
    assert sorted(tok[:4 * n_sel].tolist()) == sorted(want_tok[:4 * n_sel].tolist())
    sm = inp.slot_map[s]
    assert np.array_equal(rows, np.where(tok >= 0, sm[np.maximum(tok, 0)], -1))


# ------------------------------------------------------------------------------------------------
# expand_selection
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("wl", [synth.TINY_DECODE, synth.PADDING_DECODE,
                                synth.custom("edge", (5, 0, 2), (3, 7, 4), select_k=4, out_width=19),
                                synth.custom("causal_e", (1,), (800,), select_k=8, chunk=23,
                                             permute_slots=True)])
@pytest.mark.parametrize("with_nsel", [True, False])
def test_expand_bit_exact(cuda, wl, with_nsel):
    inp = synth.generate(wl)
    rng = np.random.default_rng(1)
    nq, S, W = len(inp.q_pos), wl.select_k, wl.out_width
    topk = np.full((nq, S), -1, np.int32)
    nsel = np.zeros(nq, np.int32)
    want_tok = np.zeros((nq, W), np.int32)
    want_rows = np.zeros((nq, W), np.int32)
    for n in range(nq):
        s = int(inp.q_seq[n])
        nv = oracle.n_visible_pools(inp.pad[s], inp.len[s], inp.q_pos[n])
        topk[n], nsel[n] = oracle.topk_pools(rng.standard_normal(nv), S)
        want_tok[n], _ = oracle.expand_selection(topk[n], nsel[n], inp.pad[s], inp.len[s], inp.q_pos[n], W)
        want_rows[n] = oracle.rows_from_tokens(want_tok[n], inp.slot_map[s])
    dims = kp.make_dims(wl.n_heads)
    tok = torch.full((nq, W), 999, dtype=torch.int32, device=cuda)
    rows = torch.full((nq, W), 999, dtype=torch.int32, device=cuda)
    kp.glm_expand_selection(dims, to_dev(topk, torch.int32, cuda), to_dev(inp.q_seq, torch.int32, cuda),
                            to_dev(inp.q_pos, torch.int32, cuda), to_dev(inp.pad, torch.int32, cuda),
                            to_dev(inp.len, torch.int32, cuda), W,
                            n_sel=to_dev(nsel, torch.int32, cuda) if with_nsel else None,
                            slot_map=to_dev(inp.slot_map, torch.int64, cuda), tok=tok, rows=rows)
    assert np.array_equal(np_(tok), want_tok)
    assert np.array_equal(np_(rows), want_rows)
    # without a slot map the rows are the tokens themselves
    rows2 = torch.full((nq, W), 999, dtype=torch.int32, device=cuda)
    kp.glm_expand_selection(dims, to_dev(topk, torch.int32, cuda), to_dev(inp.q_seq, torch.int32, cuda),
                            to_dev(inp.q_pos, torch.int32, cuda), to_dev(inp.pad, torch.int32, cuda),
                            to_dev(inp.len, torch.int32, cuda), W, rows=rows2)
    assert np.array_equal(np_(rows2), want_tok)


# ------------------------------------------------------------------------------------------------
# sparse MLA
# ------------------------------------------------------------------------------------------------

def _mla_case(cuda, n_heads, rows, cache, q, sm):
    nq, W = rows.shape
    dims = kp.make_dims(n_heads)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, nq, width=W), dtype=torch.uint8,
                     device=cuda)
    ws.fill_(0xFF)                                       # NaN-filled scratch must not leak through
    out = torch.full((nq, n_heads, 512), 7.0, dtype=torch.bfloat16, device=cuda)
    o32 = torch.full((nq, n_heads, 512), 7.0, dtype=torch.float32, device=cuda)
    lse = torch.full((nq, n_heads), 7.0, dtype=torch.float32, device=cuda)
    kp.glm_sparse_mla_decode(dims, to_dev(q, torch.bfloat16, cuda), torch.from_numpy(cache).to(cuda),
                             to_dev(rows, torch.int32, cuda), sm, out, ws, lse=lse, out_f32=o32)
    return np_(out.view(torch.int16)).view(np.uint16), np_(o32), np_(lse)


@pytest.mark.parametrize("n_heads,W,n_valid,n_rows", [(16, 80, 64, 512), (64, 2176, 2048, 5000),
                                                      (64, 2176, 2051, 3000), (128, 67, 67, 100),
                                                      (64, 1, 1, 10), (16, 300, 0, 10),
                                                      (64, 200, 3, 50), (16, 1000, 999, 5000)])
def test_sparse_mla_matches_oracle(cuda, n_heads, W, n_valid, n_rows):
    rng = np.random.default_rng(W + n_heads)
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    lat[rng.random(n_rows) < 0.01] = synth.f32_to_bf16_bits(rng.standard_normal((1, 512)).astype(np.float32) * 8)
    cache = np.zeros((n_rows, 528), np.int8)
    oracle.store_int8(lat, np.arange(n_rows, dtype=np.int64), cache)
    nq = 3
    rows = np.full((nq, W), -1, np.int32)
    for n in range(nq):
        r = rng.choice(n_rows, size=min(n_valid, n_rows), replace=False).astype(np.int32)
        pos = rng.choice(W, size=len(r), replace=False) if n == 1 else np.arange(len(r))
        rows[n, pos] = r                                # query 1 has the -1 entries interleaved
    q = synth.f32_to_bf16_bits(rng.standard_normal((nq, n_heads, 512)).astype(np.float32))
    sm = float(np.float32(512 ** -0.5))
    og, o32, lg = _mla_case(cuda, n_heads, rows, cache, q, sm)
    for n in range(nq):
        oo, lo = oracle.sparse_mla(q[n], cache, rows[n], sm)
        assert_attention_close(o32[n], oo, "f32")
        assert_bf16_is_rounded_f32(og[n], o32[n])
        if n_valid == 0:
            assert np.isneginf(lg[n]).all() and not o32[n].any() and not (og[n] & 0x7fff).any()
        else:
            np.testing.assert_allclose(lg[n], lo, atol=1e-3, rtol=0)


@pytest.mark.parametrize("fmt", ["int8", "fp8", "fp4"])
@pytest.mark.parametrize("nq", [24, 300])
def test_sparse_mla_many_queries_matches_oracle(cuda, fmt, nq):
    """24 queries: the split plan with all 64 heads of a query per CTA (one partial per 64-entry
    chunk, then the combine). 300 queries (at least two per SM): the walking plan, each CTA taking
    a run of chunks with its running softmax state in tensor memory; every fifth query's entries
    come in ascending order of row scale (latent magnitude) and some rows are 8x and 64x outliers, so that
    both references move and the accumulator is rescaled; queries are checked on a sample."""
    rng = np.random.default_rng(77 + ["int8", "fp8", "fp4"].index(fmt) + nq)
    n_heads, W, n_rows = 64, 2176, 4000
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    lat[rng.random(n_rows) < 0.01] = synth.f32_to_bf16_bits(rng.standard_normal((1, 512)).astype(np.float32) * 8)
    lat[rng.random(n_rows) < 0.005] = synth.f32_to_bf16_bits(rng.standard_normal((1, 512)).astype(np.float32) * 64)
    mag = np.abs(synth.bf16_bits_to_f32(lat)).max(axis=1)
    cache = np.zeros((n_rows, 304 if fmt == "fp4" else 528), np.int8 if fmt == "int8" else np.uint8)
    {"int8": oracle.store_int8, "fp8": oracle.store_fp8, "fp4": oracle.store_fp4}[fmt](
        lat, np.arange(n_rows, dtype=np.int64), cache)
    rows = np.full((nq, W), -1, np.int32)
    for n in range(nq):
        nv = [2051, 0, 5, 1000, 64, 2176][n % 6]
        r = rng.choice(n_rows, size=nv, replace=False).astype(np.int32)
        pos = rng.choice(W, size=nv, replace=False) if n % 2 else np.arange(nv)
        if n % 5 == 0:   # entries in ascending order of latent magnitude
            pos = np.sort(pos)
            r = r[np.argsort(mag[r], kind="stable")]
        rows[n, pos] = r
    q = synth.f32_to_bf16_bits(rng.standard_normal((nq, n_heads, 512)).astype(np.float32))
    q[3] = synth.f32_to_bf16_bits(rng.standard_normal((n_heads, 512)).astype(np.float32) * 1e-3)
    sm = float(np.float32(512 ** -0.5))
    dims = kp.make_dims(n_heads)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, nq, width=W), dtype=torch.uint8,
                     device=cuda)
    ws.fill_(0xFF)
    out = torch.full((nq, n_heads, 512), 7.0, dtype=torch.bfloat16, device=cuda)
    o32 = torch.full((nq, n_heads, 512), 7.0, dtype=torch.float32, device=cuda)
    lse = torch.full((nq, n_heads), 7.0, dtype=torch.float32, device=cuda)
    fn = {"int8": kp.glm_sparse_mla_decode, "fp8": kp.glm_sparse_mla_decode_fp8,
          "fp4": kp.glm_sparse_mla_decode_fp4}[fmt]
    fn(dims, to_dev(q, torch.bfloat16, cuda), torch.from_numpy(cache).to(cuda), to_dev(rows, torch.int32, cuda), sm,
       out, ws, lse=lse, out_f32=o32)
    og, g32, lg = np_(out.view(torch.int16)).view(np.uint16), np_(o32), np_(lse)
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    check = range(nq) if nq <= 24 else sorted(set(range(0, nq, 7)) | {1, 3, 5, nq - 1})
    for n in range(nq):
        assert_bf16_is_rounded_f32(og[n], g32[n])
    for n in check:
        if not (rows[n] >= 0).any():
            assert np.isneginf(lg[n]).all() and not g32[n].any()
            continue
        if fmt != "int8":
            c = (oracle.dequant_rows_fp8 if fmt == "fp8" else oracle.dequant_rows_fp4)(cache, rows[n][rows[n] >= 0])
            assert_attention_close(g32[n], oracle.attention_f64(qf[n], c, c, sm, shared=True), f"query {n}")
            continue
        oo, lo = oracle.sparse_mla(q[n], cache, rows[n], sm)
        assert_attention_close(g32[n], oo, f"query {n}")
        np.testing.assert_allclose(lg[n], lo, atol=1e-3, rtol=0)


def test_sparse_mla_skips_out_of_range_rows(cuda):
    rng = np.random.default_rng(5)
    n_rows = 64
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    cache = np.zeros((n_rows, 528), np.int8)
    oracle.store_int8(lat, np.arange(n_rows, dtype=np.int64), cache)
    rows = np.array([[3, 64, 9, 1 << 30, -5, 17, 63]], np.int32)   # 64 and 1<<30 are past the cache
    q = synth.f32_to_bf16_bits(rng.standard_normal((1, 16, 512)).astype(np.float32))
    sm = float(np.float32(512 ** -0.5))
    _, o32, lg = _mla_case(cuda, 16, rows, cache, q, sm)
    clean = np.where((rows >= 0) & (rows < n_rows), rows, -1)
    oo, lo = oracle.sparse_mla(q[0], cache, clean[0], sm)
    assert_attention_close(o32[0], oo)


# ------------------------------------------------------------------------------------------------
# the whole chain
# ------------------------------------------------------------------------------------------------

def _run_chain(cuda, inp):
    b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True)
    sdev.load(inp, b, build_prefix=True)
    for t in (b.topk, b.tok, b.rows):
        t.fill_(4242)
    b.out.fill_(3.0)
    P.run_step(b)
    torch.cuda.synchronize()
    return b


def _check_chain(inp, b, queries=None, check_cache_rows=None):
    """Compare a GPU step with the oracle's step on the same inputs (oracle state built by the
    oracle itself). Returns the number of queries whose selection differed inside the tie band."""
    cache_o = oracle.build_cache(inp)
    pools_o = oracle.build_pools(inp)
    cg = np_(b.cache)
    if check_cache_rows is None:
        assert np.array_equal(cg, cache_o)
    else:
        assert np.array_equal(cg[check_cache_rows], cache_o[check_cache_rows])
    pg = np_(b.pooled)
    for s, po in enumerate(pools_o):
        _pooled_close(pg[s, :po.shape[0]], po)
    sg, tg, ng, tokg, rowg = np_(b.scores), np_(b.topk), np_(b.n_sel), np_(b.tok), np_(b.rows)
    o32 = np_(b.out_f32)
    diffs = 0
    for n in (range(len(inp.q_pos)) if queries is None else queries):
        r = oracle.decode_query(inp, n, cache_o, pools_o)
        nv = r["n_vis"]
        assert score_rel_err(sg[n, :nv], r["scores"]) <= 1e-4
        assert ng[n] == r["n_sel"]
        d = _selection_agrees(tg[n], r["topk"], r["scores"], r["n_sel"])
        assert_bf16_is_rounded_f32(np_(b.out[n].view(torch.int16)).view(np.uint16), o32[n])
        if np.array_equal(tg[n], r["topk"]):
            assert np.array_equal(tokg[n], r["tok"]) and np.array_equal(rowg[n], r["rows"])
            assert_attention_close(o32[n], r["out"], f"query {n}")
            continue
        if d == 0:
            _expanded_is_valid(tokg[n], rowg[n], tg[n], r["n_sel"], r["tok"], inp, n)
        diffs += d > 0
        # a selection that differs inside the tie band (or only in the order of near-equal pools):
        # the GPU's expansion must be exactly the oracle's expansion of the GPU's own top-k, and
        # its attention the oracle's attention over the GPU's own rows
        s = int(inp.q_seq[n])
        tok_o, _ = oracle.expand_selection(tg[n], r["n_sel"], inp.pad[s], inp.len[s], inp.q_pos[n],
                                           tokg.shape[1])
        assert np.array_equal(tokg[n], tok_o)
        assert np.array_equal(rowg[n], oracle.rows_from_tokens(tok_o, inp.slot_map[s]))
        out_o, _ = oracle.sparse_mla(inp.q[n], cache_o, rowg[n], inp.sm_scale)
        assert_attention_close(o32[n], out_o, f"query {n} (own selection)")
    return diffs


@pytest.mark.parametrize("wl", [synth.TINY_DECODE, synth.PADDING_DECODE,
                                synth.custom("batched_small", (0, 0, 0, 0), (9000, 4099, 20000, 33),
                                             n_heads=64, select_k=512, out_width=2176,
                                             permute_slots=True, seed=33),
                                synth.custom("prefill_small", (0,), (6000,), n_heads=64, select_k=128,
                                             out_width=515, chunk=300, seed=44)])
def test_decode_step_matches_oracle(cuda, wl):
    inp = synth.generate(wl)
    b = _run_chain(cuda, inp)
    assert _check_chain(inp, b) <= max(1, len(inp.q_pos) // 10)


@pytest.mark.parametrize("wl", [synth.PADDING_DECODE,
                                synth.custom("batched_small2", (0, 0, 0, 0), (9000, 4099, 20000, 33),
                                             n_heads=64, select_k=512, out_width=2176,
                                             permute_slots=True, seed=37)])
def test_one_call_step_equals_separate_calls(cuda, wl):
    # glm_dsa_decode_step (fused kernels) against the separate entry points on the same inputs:
    # identical integers and identical attention
    inp = synth.generate(wl)
    outs = []
    for runner in (P.run_stages, P.run_step):
        b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True)
        sdev.load(inp, b, build_prefix=True)
        b.ws_step.fill_(0xA5)
        b.ws_step[-256:].zero_()
        runner(b)
        torch.cuda.synchronize()
        outs.append(b)
    a, c = outs
    assert int(c.ws_step[-256:-252].view(torch.int32).item()) == 0
    for name in ("cache", "pooled", "scores", "topk", "n_sel", "tok", "rows"):
        assert torch.equal(getattr(a, name), getattr(c, name)), name
    assert np.array_equal(np_(c.out_f32), np_(a.out_f32))
    assert_bf16_is_rounded_f32(np_(c.out.view(torch.int16)).view(np.uint16), np_(c.out_f32))
    assert np.array_equal(np_(a.lse), np_(c.lse))


def test_separate_calls_match_oracle(cuda):
    inp = synth.generate(synth.PADDING_DECODE)
    b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True)
    sdev.load(inp, b, build_prefix=True)
    for t in (b.topk, b.tok, b.rows):
        t.fill_(4242)
    P.run_stages(b)
    torch.cuda.synchronize()
    assert _check_chain(inp, b) <= 1


def test_long_decode_full_size(cuda):
    # the benchmark's workload and launch configuration: 262,144-token context, 65,536 pools
    inp = synth.generate(synth.LONG_DECODE)
    b = _run_chain(cuda, inp)
    assert _check_chain(inp, b) == 0


def test_batched_decode_full_size(cuda):
    inp = synth.generate(synth.BATCHED_DECODE)
    b = _run_chain(cuda, inp)
    rng = np.random.default_rng(0)
    rows = rng.choice(inp.n_rows, size=20000, replace=False)
    assert _check_chain(inp, b, check_cache_rows=rows) <= 1


def test_chunked_prefill_sampled(cuda):
    inp = synth.generate(synth.CHUNKED_PREFILL)
    b = _run_chain(cuda, inp)
    rows = np.concatenate([np.arange(131072 - 8, 135168), np.arange(0, 4096, 37)])
    # 72 of the 4,096 queries: the first four, the last, and 67 spread evenly in between
    queries = sorted(set([0, 1, 2, 3, 4095] + list(range(61, 4095, 61))))
    assert len(queries) >= 64
    assert _check_chain(inp, b, queries=queries, check_cache_rows=rows) <= len(queries) // 10
