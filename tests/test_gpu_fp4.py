"""GPU parity of the 4-bit latent cache (the opt-in 4-bit latent cache of "GLM on CUDA"; E2M1 codes, an
E4M3 scale per 16 values and an fp32 scale per row in a 304-byte row) against the oracle.

* glm_kv_store_fp4 must write exactly the oracle's bytes (code pairs, block scales, row scale, zero
  tail) and leave padding slots untouched: both sides take every rounding decision on the same
  IEEE fp32 quotients (nearest E4M3 / E2M1 value, ties to the even code, saturating, the sign kept).
* glm_sparse_mla_decode_fp4 on rows the oracle stored must match the oracle's attention over the
  same dequantised rows (value(code) value(e_k) s_row) within the attention tolerance of the INT8
  path; the one-call step on a 4-bit cache must equal the separate calls.
"""
import json
import os

import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth
from tests.conftest import GOLDEN
from tests.test_gpu_parity import assert_attention_close, assert_bf16_is_rounded_f32, np_, to_dev

pytestmark = pytest.mark.gpu

ROW = kp.GLM_FP4_ROW_BYTES


def _latents(rng, n_rows):
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    big = rng.random(n_rows) < 0.05
    lat[big] = synth.f32_to_bf16_bits((rng.standard_normal((int(big.sum()), 512)) * 8).astype(np.float32))
    return lat


def _edge_rows():
    """Rows whose blocks sit on rounding ties of both conversions (s_row = 1: amax = 2688)."""
    rows = []
    g = json.load(open(os.path.join(GOLDEN, "store_fp4_row.json")))
    x = np.zeros(512, np.float32)
    for k, v in g["nonzero"].items():
        x[int(k)] = v
    rows.append(x)
    x = np.zeros(512, np.float32)
    x[0] = 2688.0
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 6.0])
    for k in range(1, 16):                          # block scale 2^j exactly: d = 2^j
        j = k - 8
        x[16 * k:16 * k + 15] = ties * 2.0 ** j
    x[16 * 16] = 102.0                              # bmax / 6 = 17: E4M3 tie between 16 and 18 -> 16
    x[16 * 17] = 114.0                              # 19: between 18 and 20 -> 20
    x[16 * 18] = 6 * 2.0 ** -10                     # 2^-10: half the smallest subnormal -> 0
    x[16 * 18 + 1] = 1e-3
    x[16 * 19] = 6 * 1.5 * 2.0 ** -10               # 1.5 x 2^-10 -> the smallest subnormal
    x[16 * 20:16 * 21] = -0.0
    x[16 * 20] = 3.0
    rows.append(x)
    return synth.f32_to_bf16_bits(np.stack(rows))


def test_store_fp4_bit_exact(cuda):
    rng = np.random.default_rng(41)
    n = 700
    lat = _latents(rng, n)
    lat[3] = 0                                                     # zero row: the amax floor
    lat[5, :] = 0x8000                                             # -0.0 everywhere
    lat[5, 7] = synth.f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    lat[6:8] = _edge_rows()
    lat[9, 32:48] = synth.f32_to_bf16_bits(np.full(16, 1e-6, np.float32))   # a block far below the row
    slots = rng.permutation(n + 40)[:n].astype(np.int64)
    slots[rng.random(n) < 0.05] = -1                               # padding entries write nothing
    slots[[3, 5, 6, 7, 9]] = np.arange(n + 40, n + 45)             # the edge rows: slots of their own
    want = np.full((n + 48, ROW), 0x5A, np.uint8)
    oracle.store_fp4(lat, slots, want)
    got = torch.full((n + 48, ROW), 0x5A, dtype=torch.uint8, device=cuda)
    kp.glm_kv_store_fp4(kp.make_dims(64), to_dev(lat, torch.bfloat16, cuda), torch.from_numpy(slots).to(cuda), got)
    torch.cuda.synchronize()
    g = np_(got)
    bad = np.nonzero((g != want).any(axis=1))[0]
    assert bad.size == 0, (bad[:5], np.nonzero(g[bad[0]] != want[bad[0]])[0][:8] if bad.size else None)


@pytest.mark.parametrize("n_heads,W,n_valid,n_rows", [(16, 80, 64, 512), (64, 2176, 2051, 3000),
                                                      (64, 200, 3, 50), (128, 67, 67, 100)])
def test_sparse_mla_fp4_matches_oracle(cuda, n_heads, W, n_valid, n_rows):
    rng = np.random.default_rng(W + 7 * n_heads)
    lat = _latents(rng, n_rows)
    cache = np.zeros((n_rows, ROW), np.uint8)
    oracle.store_fp4(lat, np.arange(n_rows, dtype=np.int64), cache)   # inputs only
    nq = 2
    rows = np.full((nq, W), -1, np.int32)
    for n in range(nq):
        r = rng.choice(n_rows, size=min(n_valid, n_rows), replace=False).astype(np.int32)
        pos = rng.choice(W, size=len(r), replace=False) if n == 1 else np.arange(len(r))
        rows[n, pos] = r
    q = synth.f32_to_bf16_bits(rng.standard_normal((nq, n_heads, 512)).astype(np.float32))
    sm = float(np.float32(512 ** -0.5))
    dims = kp.make_dims(n_heads)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, nq, width=W), dtype=torch.uint8,
                     device=cuda)
    ws.fill_(0xFF)
    out = torch.full((nq, n_heads, 512), 7.0, dtype=torch.bfloat16, device=cuda)
    o32 = torch.full((nq, n_heads, 512), 7.0, dtype=torch.float32, device=cuda)
    lse = torch.full((nq, n_heads), 7.0, dtype=torch.float32, device=cuda)
    kp.glm_sparse_mla_decode_fp4(dims, to_dev(q, torch.bfloat16, cuda), torch.from_numpy(cache).to(cuda),
                                 to_dev(rows, torch.int32, cuda), sm, out, ws, lse=lse, out_f32=o32)
    torch.cuda.synchronize()
    g32, gb, gl = np_(o32), np_(out.view(torch.int16)).view(np.uint16), np_(lse)
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    for n in range(nq):
        valid = rows[n][rows[n] >= 0]
        c = oracle.dequant_rows_fp4(cache, valid)
        want = oracle.attention_f64(qf[n], c, c, sm, shared=True)
        assert_attention_close(g32[n], want, "fp4")
        assert_bf16_is_rounded_f32(gb[n], g32[n])
        s = (qf[n] @ c.T) * sm                                     # the log-sum-exp of the scores
        m = s.max(axis=1)
        np.testing.assert_allclose(gl[n], m + np.log(np.exp(s - m[:, None]).sum(axis=1)), atol=1e-3, rtol=0)


def test_sparse_mla_fp4_on_edge_rows(cuda):
    # rows built on rounding ties and tiny block scales, attended by a query that weights them
    lat = np.concatenate([_edge_rows(), _latents(np.random.default_rng(3), 62)])
    n_rows = lat.shape[0]
    cache = np.zeros((n_rows, ROW), np.uint8)
    oracle.store_fp4(lat, np.arange(n_rows, dtype=np.int64), cache)
    rng = np.random.default_rng(8)
    q = synth.f32_to_bf16_bits((rng.standard_normal((1, 64, 512)) * 0.05).astype(np.float32))
    rows = np.arange(n_rows, dtype=np.int32)[None]
    dims = kp.make_dims(64)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, 1, width=n_rows), dtype=torch.uint8,
                     device=cuda)
    o32 = torch.empty((1, 64, 512), dtype=torch.float32, device=cuda)
    out = torch.empty((1, 64, 512), dtype=torch.bfloat16, device=cuda)
    kp.glm_sparse_mla_decode_fp4(dims, to_dev(q, torch.bfloat16, cuda), torch.from_numpy(cache).to(cuda),
                                 to_dev(rows, torch.int32, cuda), 512 ** -0.5, out, ws, out_f32=o32)
    torch.cuda.synchronize()
    c = oracle.dequant_rows_fp4(cache, rows[0])
    qf = synth.bf16_bits_to_f32(q[0]).astype(np.float64)
    want = oracle.attention_f64(qf, c, c, float(np.float32(512 ** -0.5)), shared=True)
    # the outputs are of the size of the rows (up to 2688): the tolerance scales with them
    g = np_(o32)[0]
    scale = max(1.0, np.abs(want).max())
    assert np.abs(g - want).max() <= 1e-2 * scale
    assert np.linalg.norm(g - want) <= 5e-3 * np.linalg.norm(want)


def test_fp4_step_equals_separate_calls_and_stores_the_oracles_rows(cuda):
    from kpool_indexer_int8_b200 import pipeline as P
    from synth import device as sdev
    inp = synth.generate(synth.PADDING_DECODE)
    outs = []
    for runner in (P.run_stages, P.run_step):
        b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True, fp4=True)
        sdev.load(inp, b, build_prefix=True)
        runner(b)
        torch.cuda.synchronize()
        outs.append(b)
    a, c = outs
    for name in ("cache", "pooled", "scores", "topk", "n_sel", "tok", "rows", "out_f32", "lse"):
        assert torch.equal(getattr(a, name), getattr(c, name)), name
    want = np.zeros(tuple(c.cache.shape), np.uint8)
    oracle.store_fp4(inp.latent, inp.slots, want)
    assert np.array_equal(np_(c.cache), want)
    rows, o32 = np_(c.rows), np_(c.out_f32)
    qf = synth.bf16_bits_to_f32(inp.q).astype(np.float64)
    for n in range(len(inp.q_pos)):
        valid = rows[n][rows[n] >= 0]
        cr = oracle.dequant_rows_fp4(want, valid)
        assert_attention_close(o32[n], oracle.attention_f64(qf[n], cr, cr, inp.sm_scale, shared=True), n)


@pytest.mark.parametrize("fmt", ["fp8", "fp4"])
def test_long_decode_full_size_on_fp8_and_fp4_rows(cuda, fmt):
    # the benchmark's long-decode workload (262,144 tokens, 65,536 pools) through the one-call step
    # with FP8 or 4-bit cache rows: every stored row equals the oracle's, the selection and
    # expansion the oracle's (the index path does not depend on the row format), the attention
    # the oracle's fp64 attention over the dequantised rows it selected
    from kpool_indexer_int8_b200 import pipeline as P
    from synth import device as sdev
    inp = synth.generate(synth.LONG_DECODE)
    b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True, fp8=fmt == "fp8", fp4=fmt == "fp4")
    sdev.load(inp, b, build_prefix=True)
    b.out_f32.fill_(3.0)
    P.run_step(b)
    torch.cuda.synchronize()
    want = np.zeros(tuple(b.cache.shape), np.uint8)
    (oracle.store_fp8 if fmt == "fp8" else oracle.store_fp4)(inp.latent, inp.slots, want)
    assert np.array_equal(np_(b.cache), want)
    ref = oracle.decode_query(inp, 0, oracle.build_cache(inp), oracle.build_pools(inp))
    assert np.array_equal(np_(b.topk)[0], ref["topk"])
    assert np.array_equal(np_(b.tok)[0], ref["tok"]) and np.array_equal(np_(b.rows)[0], ref["rows"])
    valid = ref["rows"][ref["rows"] >= 0]
    c = (oracle.dequant_rows_fp8 if fmt == "fp8" else oracle.dequant_rows_fp4)(want, valid)
    qf = synth.bf16_bits_to_f32(inp.q[0]).astype(np.float64)
    assert_attention_close(np_(b.out_f32)[0], oracle.attention_f64(qf, c, c, inp.sm_scale, shared=True), fmt)
