"""Pins of the oracle's indexer steps (CPU only).

"Module glm5next_dsa_ref": layer_norm, pool_states, visible, index_scores, topk_pools,
expand_selection, and the traps (LayerNorm with bias; softmax over the pool-slot axis; pools start
at the first valid token; a pool exists only if all kpool slots are valid; -1 sentinel and a fully
written destination).
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from synth import f32_to_bf16_bits, bf16_bits_to_f32
from tests.conftest import GOLDEN

D = 128


# ------------------------------------------------------------------------------------------------
# layer_norm
# ------------------------------------------------------------------------------------------------

def test_layer_norm_golden():
    g = json.load(open(os.path.join(GOLDEN, "layer_norm_4.json")))
    for c in g["cases"]:
        y = oracle.layer_norm(g["x"], c["w"], c["b"], g["eps"])
        want = np.array(c["y_times_sqrt5"]) / np.sqrt(5.0) + np.array(c["y_offset"])
        np.testing.assert_allclose(y, want, rtol=0, atol=1e-15)


def test_layer_norm_closed_forms():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(D) * 3 + 1.5
    eps = 1e-5
    y = oracle.layer_norm(x, np.ones(D), np.zeros(D), eps)
    assert abs(y.mean()) < 1e-14
    var = x.var()
    np.testing.assert_allclose((y ** 2).mean(), var / (var + eps), rtol=1e-13)
    # a constant input gives exactly the bias
    b = rng.standard_normal(D)
    assert np.array_equal(oracle.layer_norm(np.full(D, 2.75), rng.standard_normal(D), b, eps), b)


# ------------------------------------------------------------------------------------------------
# visibility, pools and tails
# ------------------------------------------------------------------------------------------------

def test_pool_layout_golden():
    g = json.load(open(os.path.join(GOLDEN, "pool_layout.json")))
    for c in g["cases"]:
        assert oracle.n_pools(c["len"]) == c["n_pools"], c["name"]
        assert oracle.n_visible_pools(c["pad"], c["len"], c["q_pos"]) == c["n_visible"], c["name"]
        n_sel = c["n_visible"]
        topk = np.arange(max(n_sel, 1), dtype=np.int32)
        W = 4 * n_sel + 3 + 5
        tok, n = oracle.expand_selection(topk, n_sel, c["pad"], c["len"], c["q_pos"], W)
        want = [t for pool in c["pools"] for t in pool] + c["tail"]
        assert list(tok[:n]) == want, c["name"]
        assert (tok[n:] == -1).all() and n == len(want), c["name"]
    s = g["selected_rows"]
    q_pos = s["pad"] + s["len"] - 1
    n_vis = oracle.n_visible_pools(s["pad"], s["len"], q_pos)
    topk, n_sel = oracle.topk_pools(np.arange(n_vis, dtype=np.float64), s["select_k"])
    tok, n = oracle.expand_selection(topk, n_sel, s["pad"], s["len"], q_pos, s["out_width"])
    assert n == s["n_valid"]
    assert sorted(tok[:n]) == list(range(s["pad"], s["pad"] + s["len"]))


def test_visible_definition_brute_force():
    for pad, ln in [(0, 7), (3, 10), (5, 1)]:
        for q_pos in range(pad, pad + ln):
            for t in range(-2, pad + ln + 3):
                want = pad <= t <= q_pos and t < pad + ln
                assert oracle.visible(pad, ln, q_pos, t) == want


def _rand_kg(rng, T):
    k = f32_to_bf16_bits(rng.standard_normal((T, D)).astype(np.float32))
    g = f32_to_bf16_bits(rng.standard_normal((T, D)).astype(np.float32))
    return k, g


def _ln_rows(k_bits, rows, ln_w, ln_b, eps):
    x = bf16_bits_to_f32(k_bits[rows]).astype(np.float64)
    return np.stack([oracle.layer_norm(r, ln_w.astype(np.float64), ln_b.astype(np.float64), eps) for r in x])


def test_pool0_is_first_four_valid_tokens():
    # left padding [P, P, A, B, C, D]: pool 0 is [A, B, C, D] (trap 3). A gate of +60 on one slot
    # makes the pool return that slot's normalised key, which identifies the token in each slot.
    rng = np.random.default_rng(1)
    k, _ = _rand_kg(rng, 6)
    ln_w = (1 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    ln_b = (0.1 * rng.standard_normal(D)).astype(np.float32)
    for s in range(4):
        g = np.zeros((6, D), dtype=np.float32)
        g[2 + s] = 60.0
        pooled = oracle.pool_states(k, f32_to_bf16_bits(g), 2, 4, ln_w, ln_b, 1e-5)
        assert pooled.shape == (1, D)
        want = _ln_rows(k, [2 + s], ln_w, ln_b, 1e-5)[0]
        np.testing.assert_allclose(pooled[0], want, rtol=0, atol=1e-20 + 1e-12 * np.abs(want).max())


def test_seven_tokens_make_one_pool():
    rng = np.random.default_rng(2)
    k, g = _rand_kg(rng, 7)
    pooled = oracle.pool_states(k, g, 0, 7, np.ones(D, np.float32), np.zeros(D, np.float32), 1e-5)
    assert pooled.shape == (1, D)


def test_slot_softmax_axis_and_weights_sum_to_one():
    rng = np.random.default_rng(3)
    ln_w = (1 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    ln_b = (0.1 * rng.standard_normal(D)).astype(np.float32)
    k, _ = _rand_kg(rng, 8)
    # (a) gates equal across the 4 slots but varying across channels: a softmax over the slot
    # axis gives weight 1/4 everywhere, so each pool is the plain mean of its normalised keys
    # (a softmax over channels would not be).
    g = np.tile(rng.standard_normal((1, D)).astype(np.float32) * 3, (8, 1))
    pooled = oracle.pool_states(k, f32_to_bf16_bits(g), 0, 8, ln_w, ln_b, 1e-5)
    for p in range(2):
        want = _ln_rows(k, list(range(4 * p, 4 * p + 4)), ln_w, ln_b, 1e-5).mean(0)
        np.testing.assert_allclose(pooled[p], want, rtol=1e-13, atol=1e-14)
    # (b) the same key in all four slots: the pool returns it whatever the gates, so the slot
    # weights sum to one per channel.
    k4 = np.tile(k[:1], (4, 1))
    _, g4 = _rand_kg(rng, 4)
    pooled = oracle.pool_states(k4, g4, 0, 4, ln_w, ln_b, 1e-5)
    np.testing.assert_allclose(pooled[0], _ln_rows(k4, [0], ln_w, ln_b, 1e-5)[0], rtol=1e-13, atol=1e-14)
    # (c) a pool depends only on its own four tokens: changing another pool's gates changes nothing
    g2 = g.copy()
    g2[4:] = rng.standard_normal((4, D)) * 5
    p2 = oracle.pool_states(k, f32_to_bf16_bits(g2), 0, 8, ln_w, ln_b, 1e-5)
    p1 = oracle.pool_states(k, f32_to_bf16_bits(g), 0, 8, ln_w, ln_b, 1e-5)
    assert np.array_equal(p1[0], p2[0]) and not np.array_equal(p1[1], p2[1])


def test_two_slot_closed_form():
    # gates (a, b, -inf-like, -inf-like) per channel: weights sigmoid(a-b), sigmoid(b-a)
    rng = np.random.default_rng(4)
    k, _ = _rand_kg(rng, 4)
    g = np.full((4, D), -200.0, dtype=np.float32)
    a = rng.standard_normal(D).astype(np.float32)
    g[0] = a
    g[1] = 0.0
    ones, zeros = np.ones(D, np.float32), np.zeros(D, np.float32)
    pooled = oracle.pool_states(k, f32_to_bf16_bits(g), 0, 4, ones, zeros, 1e-5)[0]
    av = bf16_bits_to_f32(f32_to_bf16_bits(a)).astype(np.float64)
    y = _ln_rows(k, [0, 1], ones, zeros, 1e-5)
    w0 = 1.0 / (1.0 + np.exp(-av))
    np.testing.assert_allclose(pooled, w0 * y[0] + (1 - w0) * y[1], rtol=1e-12, atol=1e-13)


def test_padding_junk_is_ignored():
    inp = synth.generate(synth.PADDING_DECODE, junk_padding=True)
    inp2 = synth.generate(synth.PADDING_DECODE, junk_padding=False)
    p1 = oracle.build_pools(inp)
    p2 = oracle.build_pools(inp2)
    for a, b in zip(p1, p2):
        assert np.array_equal(a, b)
    assert [p.shape[0] for p in p1] == [1, 16, 256, 1024]


# ------------------------------------------------------------------------------------------------
# index_scores
# ------------------------------------------------------------------------------------------------

def _qw(rng, H=32):
    q = f32_to_bf16_bits(rng.standard_normal((H, D)).astype(np.float32))
    w = rng.random(H, dtype=np.float32)
    return q, w


def test_scores_all_negative_dots_are_exactly_zero():
    rng = np.random.default_rng(5)
    q = f32_to_bf16_bits(np.abs(rng.standard_normal((32, D))).astype(np.float32))
    pooled = -np.abs(rng.standard_normal((10, D)))
    s = oracle.index_scores(q, rng.random(32, dtype=np.float32), pooled, 10)
    assert np.array_equal(s, np.zeros(10))


def test_scores_one_hot_weight_is_one_relu_dot():
    rng = np.random.default_rng(6)
    q, _ = _qw(rng)
    pooled = rng.standard_normal((20, D))
    qv = bf16_bits_to_f32(q).astype(np.float64)
    for h in (0, 17, 31):
        w = np.zeros(32, np.float32)
        w[h] = 1.0
        s = oracle.index_scores(q, w, pooled, 20)
        np.testing.assert_allclose(s, np.maximum(pooled @ qv[h], 0.0), rtol=1e-13, atol=1e-13)


def test_scores_unit_vector_queries_closed_form():
    # q_h = e_{d(h)}: the dot is pooled[p, d(h)], so score = sum_h w_h relu(pooled[p, d(h)]).
    # A transposed operand or a wrong head/dim index fails this.
    rng = np.random.default_rng(8)
    dh = rng.permutation(D)[:32]
    qf = np.zeros((32, D), np.float32)
    qf[np.arange(32), dh] = 1.0
    w = rng.random(32, dtype=np.float32)
    pooled = rng.standard_normal((9, D))
    s = oracle.index_scores(f32_to_bf16_bits(qf), w, pooled, 9)
    want = (np.maximum(pooled[:, dh], 0.0) * w.astype(np.float64)).sum(1)
    np.testing.assert_allclose(s, want, rtol=1e-14, atol=1e-15)


def test_scores_scale_with_weights_and_only_visible_pools():
    rng = np.random.default_rng(9)
    q, w = _qw(rng)
    pooled = rng.standard_normal((12, D))
    s1 = oracle.index_scores(q, w, pooled, 12)
    s2 = oracle.index_scores(q, (w * 2).astype(np.float32), pooled, 12)
    assert np.array_equal(s2, 2 * s1)
    s3 = oracle.index_scores(q, w, pooled, 5)
    assert s3.shape == (5,) and np.array_equal(s3, s1[:5])


# ------------------------------------------------------------------------------------------------
# topk_pools
# ------------------------------------------------------------------------------------------------

def test_topk_golden():
    g = json.load(open(os.path.join(GOLDEN, "topk_small.json")))
    for c in g["cases"]:
        ids, n_sel = oracle.topk_pools(np.array(c["scores"], dtype=np.float64), c["select_k"])
        assert list(ids) == c["ids"] and n_sel == c["n_sel"], c


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(10)
    for trial in range(50):
        n = int(rng.integers(0, 60))
        s = rng.integers(0, 8, size=n).astype(np.float64) * 0.25   # many ties
        if n:
            s[rng.random(n) < 0.1] = -0.0
        S = int(rng.integers(1, 40))
        ids, n_sel = oracle.topk_pools(s, S)
        order = sorted(range(n), key=lambda i: (-s[i], i))
        want = order[:S] + [-1] * max(0, S - n)
        assert list(ids) == want and n_sel == min(S, n)


def test_topk_all_equal_picks_lowest_ids():
    ids, n_sel = oracle.topk_pools(np.full(100, 3.5), 16)
    assert list(ids) == list(range(16)) and n_sel == 16


# ------------------------------------------------------------------------------------------------
# expand_selection
# ------------------------------------------------------------------------------------------------

def test_expand_order_count_and_full_write():
    rng = np.random.default_rng(12)
    pad, ln = 3, 1027
    q_pos = pad + ln - 1
    n_vis = oracle.n_visible_pools(pad, ln, q_pos)
    assert n_vis == 256
    scores = rng.standard_normal(n_vis)
    topk, n_sel = oracle.topk_pools(scores, 512)
    tok, n = oracle.expand_selection(topk, n_sel, pad, ln, q_pos, 2176)
    assert n == 4 * n_sel + 3 == 1027
    assert (tok[n:] == -1).all()
    assert sorted(tok[:n]) == list(range(pad, pad + ln))          # every visible token once
    for i in range(n_sel):                                          # pools in top-k order
        assert list(tok[4 * i:4 * i + 4]) == [pad + 4 * topk[i] + s for s in range(4)]
    assert list(tok[4 * n_sel:n]) == [1027, 1028, 1029]


def test_expand_too_narrow_is_an_error():
    topk = np.arange(4, dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.expand_selection(topk, 4, 0, 19, 18, 18)        # needs 16 + 3
    tok, n = oracle.expand_selection(topk, 4, 0, 19, 18, 19)
    assert n == 19


def test_expand_selected_subset_when_many_pools():
    rng = np.random.default_rng(13)
    pad, ln = 0, 4096
    q_pos = ln - 1
    n_vis = oracle.n_visible_pools(pad, ln, q_pos)
    scores = rng.standard_normal(n_vis)
    topk, n_sel = oracle.topk_pools(scores, 512)
    tok, n = oracle.expand_selection(topk, n_sel, pad, ln, q_pos, 2176)
    assert n_sel == 512 and n == 2048
    # the selected tokens are exactly the tokens of the 512 highest-scoring pools
    best = np.argsort(-scores, kind="stable")[:512]
    assert set(tok[:n].tolist()) == {4 * p + s for p in best.tolist() for s in range(4)}
    assert (tok[n:] == -1).all()


def test_rows_through_slot_map():
    tok = np.array([0, 2, -1, 5], dtype=np.int32)
    slot_map = np.array([10, -1, 30, 40, 50, 60], dtype=np.int64)
    assert list(oracle.rows_from_tokens(tok, slot_map)) == [10, 30, -1, 60]
