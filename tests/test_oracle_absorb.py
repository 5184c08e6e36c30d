"""Pins of the oracle's MLA up-projection (CPU only).

"Module glm5next_dsa_ref", expand_kv: the compressed latent is expanded into per-head K and V by
kv_b_proj ("linear": y = x @ w^T); "GLM-5.3-Flash" 'Checkpoint shape': 64 heads, kv_lora_rank 512,
qk_head_dim = v_head_dim = 256, no RoPE. The sparse MLA of this path works in latent space (the
latent is both K and V); its output meets the expanded form through two identities,
q_h . K_h,t = (q_h W_k,h) . c_t and sum_t p_t V_h,t = (sum_t p_t c_t) W_v,h^T, which the first test
checks with independent oracle functions on each side. The other tests fix each function's
indexing by weights with a known answer.
"""
import numpy as np
import pytest

import oracle
from synth import bf16_bits_to_f32, f32_to_bf16_bits


def _bf16_weights(rng, n_heads, dk, dv, latent=512, std=0.05):
    return f32_to_bf16_bits((rng.standard_normal((n_heads * (dk + dv), latent)) * std).astype(np.float32))


def _bf16_values(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


@pytest.mark.parametrize("n_heads,dk,dv,T", [(4, 32, 24, 20), (2, 256, 256, 9)])
def test_absorbed_form_equals_expanded_form(n_heads, dk, dv, T):
    rng = np.random.default_rng(11 + dk)
    w = _bf16_weights(rng, n_heads, dk, dv)
    c = rng.standard_normal((T, 512))
    q = rng.standard_normal((n_heads, dk))
    scale = dk ** -0.5
    k, v = oracle.expand_kv(c, w, n_heads, dk, dv)
    expanded = oracle.attention_f64(q, k, v, scale, shared=False)
    o_lat = oracle.attention_f64(oracle.q_absorb(q, w, dk, dv), c, c, scale, shared=True)
    absorbed = oracle.v_up(o_lat, w, dk, dv)
    assert absorbed.shape == expanded.shape == (n_heads, dv)
    assert np.allclose(absorbed, expanded, rtol=1e-11, atol=1e-13)


def test_expand_kv_reads_each_heads_rows():
    # K row e of head h a unit vector at dim (7 h + e) % 512, V row e at (300 + 5 h + 3 e) % 512:
    # K and V are those latent columns exactly (a transposed weight, a wrong head offset or a V
    # row read from the K half would all show)
    n_heads, dk, dv, T = 3, 4, 5, 6
    w = np.zeros((n_heads * (dk + dv), 512), dtype=np.float32)
    for h in range(n_heads):
        for e in range(dk):
            w[h * (dk + dv) + e, (7 * h + e) % 512] = 1.0
        for e in range(dv):
            w[h * (dk + dv) + dk + e, (300 + 5 * h + 3 * e) % 512] = 1.0
    c = np.random.default_rng(3).standard_normal((T, 512))
    k, v = oracle.expand_kv(c, f32_to_bf16_bits(w), n_heads, dk, dv)
    for h in range(n_heads):
        assert np.array_equal(k[h], c[:, [(7 * h + e) % 512 for e in range(dk)]])
        assert np.array_equal(v[h], c[:, [(300 + 5 * h + 3 * e) % 512 for e in range(dv)]])


def test_v_up_is_a_per_head_row_selection_for_one_hot_weights():
    n_heads, dk, dv = 4, 6, 8
    rng = np.random.default_rng(4)
    w = rng.standard_normal((n_heads * (dk + dv), 512)).astype(np.float32)   # K half: noise
    perm = [rng.permutation(512)[:dv] for _ in range(n_heads)]
    for h in range(n_heads):
        w[h * (dk + dv) + dk:(h + 1) * (dk + dv)] = 0.0
        for e in range(dv):
            w[h * (dk + dv) + dk + e, perm[h][e]] = 1.0
    o_lat = rng.standard_normal((n_heads, 512))
    out = oracle.v_up(o_lat, f32_to_bf16_bits(w), dk, dv)
    for h in range(n_heads):
        assert np.array_equal(out[h], o_lat[h, perm[h]])


def test_q_absorb_is_q_times_the_k_rows():
    # with W_k,h = s_h * [I_dk | 0] (the first dk latent dims, scaled per head) q_lat = s_h q, padded
    n_heads, dk, dv = 3, 5, 2
    w = np.zeros((n_heads * (dk + dv), 512), dtype=np.float32)
    for h in range(n_heads):
        for e in range(dk):
            w[h * (dk + dv) + e, e] = 2.0 ** h
        w[h * (dk + dv) + dk:(h + 1) * (dk + dv), :] = 3.0                    # V half: must not be read
    q = np.random.default_rng(5).standard_normal((n_heads, dk))
    ql = oracle.q_absorb(q, f32_to_bf16_bits(w), dk, dv)
    for h in range(n_heads):
        assert np.array_equal(ql[h, :dk], q[h] * 2.0 ** h)
        assert not ql[h, dk:].any()


def test_attention_closed_forms():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((5, 16))
    v = rng.standard_normal((5, 7))
    q = rng.standard_normal((3, 16))
    # one key: the output is its value
    assert np.array_equal(oracle.attention_f64(q, k[:1], v[:1], 0.3, shared=True), np.tile(v[0], (3, 1)))
    # a zero query (equal scores): the mean of the values
    assert np.allclose(oracle.attention_f64(np.zeros((1, 16)), k, v, 0.3, shared=True)[0], v.mean(axis=0),
                       rtol=1e-14, atol=1e-15)
    # two keys: the sigmoid weights of the score difference
    s = 0.3 * (q @ k[:2].T)
    p1 = 1.0 / (1.0 + np.exp(s[:, 0] - s[:, 1]))
    want = (1 - p1)[:, None] * v[0] + p1[:, None] * v[1]
    assert np.allclose(oracle.attention_f64(q, k[:2], v[:2], 0.3, shared=True), want, rtol=1e-13, atol=1e-14)


def test_latent_attention_is_the_sparse_mla_on_the_same_rows():
    # attention_f64 in latent form (K = V = the dequantised rows) against the sparse MLA (pinned on
    # its own) on the same rows and bf16 queries
    rng = np.random.default_rng(8)
    n_rows, Hm = 12, 4
    lat = f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    cache = np.zeros((n_rows, 528), np.int8)
    oracle.store_int8(lat, np.arange(n_rows, dtype=np.int64), cache)
    rows = np.array([3, 0, 11, 7, 7, 5], dtype=np.int32)
    q = f32_to_bf16_bits(rng.standard_normal((Hm, 512)).astype(np.float32))
    want, _ = oracle.sparse_mla(q, cache, rows, 512 ** -0.5)
    c = oracle.dequant_rows(cache, rows)
    got = oracle.attention_f64(_bf16_values(q), c, c, 512 ** -0.5, shared=True)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)
