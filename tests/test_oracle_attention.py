"""Pins of the oracle's sparse NoPE MLA over int8 rows (CPU only).

"GLM-5.3 Kernels" README, titan_mla.triton_mla_sparse_attention (shared 512-d latent as K and V,
fp32 softmax/accumulation) and 'Measurements and validation' (INT8 MLA vs BF16 source latents:
output NMSE about 4.97e-5, cosine about 0.999975); "Module glm5next_dsa_ref" topk_to_mask and
mla_masked_attention.
"""
import numpy as np

import oracle
import synth
from synth import f32_to_bf16_bits, bf16_bits_to_f32

ROW = 528
SM = float(np.float32(512 ** -0.5))


def _cache(rng, n, scale=1.0):
    lat = f32_to_bf16_bits((rng.standard_normal((n, 512)) * scale).astype(np.float32))
    cache = np.zeros((n, ROW), dtype=np.int8)
    oracle.store_int8(lat, np.arange(n, dtype=np.int64), cache)
    return lat, cache


def _q(rng, H):
    return f32_to_bf16_bits(rng.standard_normal((H, 512)).astype(np.float32))


def test_single_row_returns_that_row():
    rng = np.random.default_rng(0)
    _, cache = _cache(rng, 10)
    q = _q(rng, 4)
    rows = np.array([-1, 7, -1, -1], dtype=np.int32)
    out, lse = oracle.sparse_mla(q, cache, rows, SM)
    c = oracle.dequant_rows(cache, [7])[0]
    for h in range(4):
        assert np.array_equal(out[h], c)
    qv = bf16_bits_to_f32(q).astype(np.float64)
    np.testing.assert_allclose(lse, SM * (qv @ c), rtol=1e-13)


def test_identical_rows_and_uniform_scores():
    rng = np.random.default_rng(1)
    _, cache = _cache(rng, 6)
    q = _q(rng, 3)
    c3 = oracle.dequant_rows(cache, [3])[0]
    out, lse = oracle.sparse_mla(q, cache, np.array([3, 3, 3], np.int32), SM)
    np.testing.assert_allclose(out, np.tile(c3, (3, 1)), rtol=1e-15, atol=1e-15)
    qv = bf16_bits_to_f32(q).astype(np.float64)
    np.testing.assert_allclose(lse, SM * (qv @ c3) + np.log(3), rtol=1e-13)
    # q = 0: uniform weights -> the mean of the rows, lse = log(n)
    rows = np.array([0, 1, 2, 4, 5], np.int32)
    out, lse = oracle.sparse_mla(np.zeros((2, 512), np.uint16), cache, rows, SM)
    np.testing.assert_allclose(out[0], oracle.dequant_rows(cache, rows).mean(0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse, np.log(5), rtol=1e-15)


def test_two_rows_closed_form():
    # o = sigmoid(s1 - s2) c1 + sigmoid(s2 - s1) c2: pins the sign and the scale of the scores
    rng = np.random.default_rng(2)
    _, cache = _cache(rng, 2, scale=0.3)
    q = _q(rng, 5)
    out, lse = oracle.sparse_mla(q, cache, np.array([0, 1], np.int32), SM)
    c = oracle.dequant_rows(cache, [0, 1])
    s = SM * (bf16_bits_to_f32(q).astype(np.float64) @ c.T)
    a = 1.0 / (1.0 + np.exp(-(s[:, 0] - s[:, 1])))
    np.testing.assert_allclose(out, a[:, None] * c[0] + (1 - a)[:, None] * c[1], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, np.logaddexp(s[:, 0], s[:, 1]), rtol=1e-13)


def test_no_valid_rows_gives_zero_and_neg_inf():
    rng = np.random.default_rng(3)
    _, cache = _cache(rng, 4)
    out, lse = oracle.sparse_mla(_q(rng, 2), cache, np.full(8, -1, np.int32), SM)
    assert not out.any() and np.isneginf(lse).all()


def test_gather_form_equals_dense_masked_form_and_is_order_free():
    rng = np.random.default_rng(4)
    T = 300
    _, cache = _cache(rng, T)
    slot_map = rng.permutation(T).astype(np.int64)   # token t lives in row slot_map[t]
    q = _q(rng, 8)
    tok = rng.choice(T, size=40, replace=False).astype(np.int32)
    tok = np.concatenate([tok, np.full(9, -1, np.int32)])
    rows = oracle.rows_from_tokens(tok, slot_map)
    out, lse = oracle.sparse_mla(q, cache, rows, SM)
    mask = oracle.topk_to_mask(tok, T)
    assert mask.sum() == 40
    out2, lse2 = oracle.masked_attention(q, cache, slot_map, mask, SM)
    np.testing.assert_allclose(out, out2, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=1e-13)
    perm = rng.permutation(len(rows))
    out3, lse3 = oracle.sparse_mla(q, cache, rows[perm], SM)
    np.testing.assert_allclose(out, out3, rtol=1e-11, atol=1e-14)


def test_int8_cache_close_to_bf16_attention():
    # Soft bound from the page's INT8-vs-BF16 comparison (NMSE about 5e-5, cosine about 0.99997):
    # attention over the int8 rows stays that close to attention over the bf16 source latents.
    rng = np.random.default_rng(5)
    n = 2048
    lat, cache = _cache(rng, n)
    q = _q(rng, 16)
    out, _ = oracle.sparse_mla(q, cache, np.arange(n, dtype=np.int32), SM)
    k = bf16_bits_to_f32(lat).astype(np.float64)
    s = SM * (bf16_bits_to_f32(q).astype(np.float64) @ k.T)
    p = np.exp(s - s.max(1, keepdims=True))
    ref = (p / p.sum(1, keepdims=True)) @ k
    nmse = ((out - ref) ** 2).sum(1) / (ref ** 2).sum(1)
    cos = (out * ref).sum(1) / np.linalg.norm(out, axis=1) / np.linalg.norm(ref, axis=1)
    assert nmse.max() < 2e-4 and cos.min() > 0.9999, (nmse.max(), cos.min())


def test_index_past_cache_is_an_error():
    rng = np.random.default_rng(6)
    _, cache = _cache(rng, 4)
    try:
        oracle.sparse_mla(_q(rng, 1), cache, np.array([4], np.int32), SM)
    except ValueError:
        return
    raise AssertionError("expected an error")


def test_end_to_end_tiny_decode_composition():
    # the whole path on the tiny workload: 128 pools, 16 selected -> 64 tokens, width 80
    inp = synth.generate(synth.TINY_DECODE)
    cache = oracle.build_cache(inp)
    pools = oracle.build_pools(inp)
    r = oracle.decode_query(inp, 0, cache, pools)
    assert r["n_vis"] == 128 and r["n_sel"] == 16 and r["n_valid"] == 64
    assert (r["tok"][64:] == -1).all() and r["tok"].shape == (80,)
    assert r["out"].shape == (16, 512) and np.isfinite(r["lse"]).all()
    # the selected pools are the 16 best by score
    best = np.argsort(-r["scores"], kind="stable")[:16]
    assert list(r["topk"]) == best.tolist()
