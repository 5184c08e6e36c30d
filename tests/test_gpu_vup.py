"""The up-projection after the absorbed MLA (glm_mla_v_up) against the fp64 oracle.

out_v[n][h][e] = sum_d o_lat[n][h][d] W[h (dk + dv) + dk + e][d] with bf16 o_lat and W: the kernel
multiplies them exactly on the tensor cores and accumulates 512 products in fp32, so each output
is within gamma_512 * sum_d |o_lat[d] W[e][d]| of the exact sum (gamma_512 = 512 u / (1 - 512 u),
u = 2^-24); the bf16 output is the fp32 output rounded to nearest even. The chain test runs the
sparse MLA on absorbed queries and up-projects its output: against the oracle's fp64 chain on the
same inputs it must hold the attention tolerance (1e-2 absolute, 5e-3 relative L2).
"""
import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth

pytestmark = pytest.mark.gpu

U = 2.0 ** -24
GAMMA_512 = 512 * U / (1 - 512 * U)


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


def _to_dev(bits, dev):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


@pytest.mark.parametrize("n_heads,dk,dv,n_q", [(64, 256, 256, 1), (64, 256, 256, 3), (16, 128, 128, 200),
                                               (32, 0, 384, 130), (64, 256, 256, 4096)])
def test_v_up_matches_oracle(n_heads, dk, dv, n_q):
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(n_heads + dk + dv + n_q)
    o_lat = _bf16(rng.standard_normal((n_q, n_heads, 512)))
    w = _bf16(rng.standard_normal((n_heads * (dk + dv), 512)) / np.sqrt(512))
    dims = kp.make_dims(n_heads)
    out = torch.full((n_q, n_heads, dv), 5.0, dtype=torch.bfloat16, device=dev)
    o32 = torch.full((n_q, n_heads, dv), 5.0, dtype=torch.float32, device=dev)
    kp.glm_mla_v_up(dims, _to_dev(o_lat, dev), _to_dev(w, dev), dk, dv, out, out_v_f32=o32)
    torch.cuda.synchronize()
    g32 = o32.cpu().numpy().astype(np.float64)
    gb = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(gb, _bf16(o32.cpu().numpy()))
    wf = synth.bf16_bits_to_f32(w).astype(np.float64).reshape(n_heads, dk + dv, 512)[:, dk:]
    # every query at small sizes; at 4,096 queries the first, the last and a spread of 64 others
    qs = range(n_q) if n_q <= 200 else sorted(set([0, n_q - 1] + list(range(1, n_q, n_q // 64))))
    for n in qs:
        a = synth.bf16_bits_to_f32(o_lat[n]).astype(np.float64)
        want = oracle.v_up(a, w, dk, dv)
        bound = GAMMA_512 * np.einsum("hd,hed->he", np.abs(a), np.abs(wf)) + 1e-30
        assert (np.abs(g32[n] - want) <= bound).all(), (n, float((np.abs(g32[n] - want) / bound).max()))


def test_v_up_after_sparse_mla_matches_the_oracle_chain():
    # per-head no-RoPE queries absorbed into the latent space, the sparse MLA over int8 rows, then the
    # up-projection: the GPU chain against the oracle's fp64 chain on the same bf16 inputs
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(3)
    n_heads, dk, dv, n_rows, width, n_q = 64, 256, 256, 3000, 2176, 2
    w = _bf16(rng.standard_normal((n_heads * (dk + dv), 512)) / np.sqrt(512))
    lat = _bf16(rng.standard_normal((n_rows, 512)))
    cache = np.zeros((n_rows, 528), np.int8)
    oracle.store_int8(lat, np.arange(n_rows, dtype=np.int64), cache)
    q_nope = rng.standard_normal((n_q, n_heads, dk))
    q_lat = np.stack([_bf16(oracle.q_absorb(q_nope[n], w, dk, dv)) for n in range(n_q)])
    rows = np.full((n_q, width), -1, np.int32)
    for n in range(n_q):
        rows[n, :2051] = rng.choice(n_rows, size=2051, replace=False)
    sm = float(np.float32(256 ** -0.5))
    dims = kp.make_dims(n_heads)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, n_q, width=width), dtype=torch.uint8,
                     device=dev)
    o_lat = torch.empty(n_q, n_heads, 512, dtype=torch.bfloat16, device=dev)
    kp.glm_sparse_mla_decode(dims, _to_dev(q_lat, dev), torch.from_numpy(cache).to(dev),
                             torch.from_numpy(rows).to(dev), sm, o_lat, ws)
    o32 = torch.empty(n_q, n_heads, dv, dtype=torch.float32, device=dev)
    out = torch.empty(n_q, n_heads, dv, dtype=torch.bfloat16, device=dev)
    kp.glm_mla_v_up(dims, o_lat, _to_dev(w, dev), dk, dv, out, out_v_f32=o32)
    torch.cuda.synchronize()
    g = o32.cpu().numpy().astype(np.float64)
    for n in range(n_q):
        lat_out, _ = oracle.sparse_mla(q_lat[n], cache, rows[n], sm)
        want = oracle.v_up(lat_out, w, dk, dv)
        err = np.abs(g[n] - want).max()
        rel = np.linalg.norm(g[n] - want) / np.linalg.norm(want)
        assert err <= 1e-2 and rel <= 5e-3, (n, err, rel)
