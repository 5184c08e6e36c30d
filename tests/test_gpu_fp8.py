"""GPU parity of the FP8 latent cache (the opt-in FP8 latent cache of "GLM on CUDA"; E4M3 codes and
one fp32 scale per row in the 528-byte layout) against the oracle.

* glm_kv_store_fp8 must write exactly the oracle's bytes (codes, scale, zero tail), and leave
  padding slots untouched: both quantise the same bf16 values with one recipe (IEEE fp32 quotient,
  nearest E4M3 value with ties to the even code, saturation at 448, the sign kept).
* glm_sparse_mla_decode_fp8 on rows the oracle stored must match the oracle's attention over the
  same dequantised rows (value(code) * scale) within the attention tolerance of the INT8 path.
"""
import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth
from tests.test_gpu_parity import assert_attention_close, assert_bf16_is_rounded_f32, np_, to_dev

pytestmark = pytest.mark.gpu


def _latents(rng, n_rows):
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    big = rng.random(n_rows) < 0.05
    lat[big] = synth.f32_to_bf16_bits((rng.standard_normal((int(big.sum()), 512)) * 8).astype(np.float32))
    return lat


def test_store_fp8_bit_exact(cuda):
    rng = np.random.default_rng(21)
    n = 700
    lat = _latents(rng, n)
    lat[3] = 0                                                     # zero row: the amax floor
    edge = np.zeros(512, np.float32)                               # exact E4M3 midpoints at scale 1
    edge[:12] = [448.0, 1.0, -2.0, 0.296875, 0.328125, 17.0, 19.0, 240.0, 0.0009765625, 0.0029296875,
                 0.0146484375, -0.0009765625]
    lat[4] = synth.f32_to_bf16_bits(edge)
    lat[5, :] = 0x8000                                             # -0.0 everywhere (the floor, signed zeros)
    lat[5, 0] = synth.f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    slots = rng.permutation(n + 40)[:n].astype(np.int64)
    slots[rng.random(n) < 0.05] = -1                               # padding entries write nothing
    want = np.full((n + 40, 528), 0x5A, np.uint8)
    oracle.store_fp8(lat, slots, want)
    got = torch.full((n + 40, 528), 0x5A, dtype=torch.uint8, device=cuda)
    kp.glm_kv_store_fp8(kp.make_dims(64), to_dev(lat, torch.bfloat16, cuda),
                        torch.from_numpy(slots).to(cuda), got)
    torch.cuda.synchronize()
    g = np_(got)
    bad = np.nonzero((g != want).any(axis=1))[0]
    assert bad.size == 0, (bad[:5], g[bad[0], :16] if bad.size else None, want[bad[0], :16] if bad.size else None)


@pytest.mark.parametrize("n_heads,W,n_valid,n_rows", [(16, 80, 64, 512), (64, 2176, 2051, 3000),
                                                      (64, 200, 3, 50), (128, 67, 67, 100)])
def test_sparse_mla_fp8_matches_oracle(cuda, n_heads, W, n_valid, n_rows):
    rng = np.random.default_rng(W + 3 * n_heads)
    lat = _latents(rng, n_rows)
    cache = np.zeros((n_rows, 528), np.uint8)
    oracle.store_fp8(lat, np.arange(n_rows, dtype=np.int64), cache)   # inputs only
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
    kp.glm_sparse_mla_decode_fp8(dims, to_dev(q, torch.bfloat16, cuda),
                                 torch.from_numpy(cache).to(cuda), to_dev(rows, torch.int32, cuda), sm, out, ws,
                                 out_f32=o32)
    torch.cuda.synchronize()
    g32, gb = np_(o32), np_(out.view(torch.int16)).view(np.uint16)
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    for n in range(nq):
        valid = rows[n][rows[n] >= 0]
        c = oracle.dequant_rows_fp8(cache, valid)
        want = oracle.attention_f64(qf[n], c, c, sm, shared=True)
        assert_attention_close(g32[n], want, "fp8")
        assert_bf16_is_rounded_f32(gb[n], g32[n])


def test_fp8_step_equals_separate_calls_and_stores_the_oracles_rows(cuda):
    # the one-call step on an FP8 cache against the separate entry points (identical integers and
    # attention), its cache against the oracle's FP8 store of every token, and its attention
    # against the oracle's over the rows it selected
    from kpool_indexer_int8_b200 import pipeline as P
    from synth import device as sdev
    inp = synth.generate(synth.PADDING_DECODE)
    outs = []
    for runner in (P.run_stages, P.run_step):
        b = sdev.allocate_for(inp, cuda, keep_scores=True, keep_f32=True, fp8=True)
        sdev.load(inp, b, build_prefix=True)
        runner(b)
        torch.cuda.synchronize()
        outs.append(b)
    a, c = outs
    for name in ("cache", "pooled", "scores", "topk", "n_sel", "tok", "rows", "out_f32", "lse"):
        assert torch.equal(getattr(a, name), getattr(c, name)), name
    want = np.zeros(tuple(c.cache.shape), np.uint8)
    oracle.store_fp8(inp.latent, inp.slots, want)
    assert np.array_equal(np_(c.cache), want)
    rows, o32 = np_(c.rows), np_(c.out_f32)
    qf = synth.bf16_bits_to_f32(inp.q).astype(np.float64)
    for n in range(len(inp.q_pos)):
        valid = rows[n][rows[n] >= 0]
        cr = oracle.dequant_rows_fp8(want, valid)
        assert_attention_close(o32[n], oracle.attention_f64(qf[n], cr, cr, inp.sm_scale, shared=True), n)
