"""The allocation-free sparse MLA entry point (glm_sparse_mla_decode_noalloc).

It serves callers that cannot allocate device memory where they run the attention (plugin
interfaces that pass only inputs and outputs; serving loops that allow no allocation after
start-up). Its split partials live in a fixed scratch array inside the library instead of a
caller workspace. Through the C ABI, calls in a row must give exactly the results of the workspace
entry point glm_sparse_mla_decode (the same kernels with the same plan run on the same data), and
those must agree with the fp64 oracle within the attention tolerance. The second call follows a
large one and has a query whose chunks are all padding and a query with no valid entry at all, so
that a partial left in the scratch by the first call would show. A request larger than the
scratch must be refused. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth

pytestmark = pytest.mark.gpu

SM = float(np.float32(512 ** -0.5))


def _inputs(seed, n_heads, n_rows, rows):
    rng = np.random.default_rng(seed)
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    cache = np.zeros((n_rows, 528), np.int8)
    oracle.store_int8(lat, np.arange(n_rows, dtype=np.int64), cache)   # inputs only
    q = synth.f32_to_bf16_bits(rng.standard_normal((rows.shape[0], n_heads, 512)).astype(np.float32))
    return q, cache


def _dev(dev, q, cache, rows):
    return (torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).to(dev), torch.from_numpy(cache).to(dev),
            torch.from_numpy(rows).to(dev))


def _workspace_result(dims, q, cache, rows):
    n_q, heads = q.shape[0], q.shape[1]
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, n_q, width=rows.shape[1]),
                     dtype=torch.uint8, device=q.device)
    out = torch.empty(n_q, heads, 512, dtype=torch.bfloat16, device=q.device)
    o32 = torch.empty(n_q, heads, 512, dtype=torch.float32, device=q.device)
    lse = torch.empty(n_q, heads, dtype=torch.float32, device=q.device)
    kp.glm_sparse_mla_decode(dims, q, cache, rows, SM, out, ws, lse=lse, out_f32=o32)
    return out, o32, lse


def _noalloc_result(dims, q, cache, rows):
    n_q, heads = q.shape[0], q.shape[1]
    out = torch.full((n_q, heads, 512), 9.0, dtype=torch.bfloat16, device=q.device)
    o32 = torch.full((n_q, heads, 512), 9.0, dtype=torch.float32, device=q.device)
    lse = torch.full((n_q, heads), 9.0, dtype=torch.float32, device=q.device)
    kp.glm_sparse_mla_decode_noalloc(dims, q, cache, rows, SM, out, lse=lse, out_f32=o32)
    return out, o32, lse


def _check(q_np, cache_np, rows_np, got, ref):
    for g, r in zip(got, ref):   # bit-identical to the workspace entry point
        assert torch.equal(g.view(torch.int16) if g.dtype == torch.bfloat16 else g.view(torch.int32),
                           r.view(torch.int16) if r.dtype == torch.bfloat16 else r.view(torch.int32))
    o32, lse = got[1].cpu().numpy().astype(np.float64), got[2].cpu().numpy()
    for n in range(rows_np.shape[0]):
        oo, lo = oracle.sparse_mla(q_np[n], cache_np, rows_np[n], SM)
        if not (rows_np[n] >= 0).any():
            assert not o32[n].any() and np.isneginf(lse[n]).all()
            continue
        max_abs = np.abs(o32[n] - oo).max()
        rel = np.linalg.norm(o32[n] - oo) / np.linalg.norm(oo)
        assert max_abs <= 1e-2 and rel <= 5e-3, (n, max_abs, rel)
        np.testing.assert_allclose(lse[n], lo, atol=1e-3, rtol=0)


def test_noalloc_matches_workspace_entry_and_oracle_on_calls_in_a_row():
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(7)
    # call 1: two 64-head queries with every entry of width 2,176 valid
    rows1 = np.stack([rng.choice(6000, size=2176, replace=False) for _ in range(2)]).astype(np.int32)
    # call 2: query 0 has valid entries in its first chunk only (the rest of its chunks are padding
    # and were full in call 1), query 1 has none, query 2 is padded in between
    rows2 = np.full((3, 2176), -1, np.int32)
    rows2[0, :37] = rng.choice(6000, size=37, replace=False)
    rows2[2, ::5] = rng.choice(6000, size=len(rows2[2, ::5]), replace=False)
    # call 3: another geometry (16 heads, width 80)
    rows3 = np.full((3, 80), -1, np.int32)
    rows3[:, :67] = np.stack([rng.choice(500, size=67, replace=False) for _ in range(3)])
    for seed, heads, n_rows, rows in ((1, 64, 6000, rows1), (2, 64, 6000, rows2), (3, 16, 500, rows3)):
        dims = kp.make_dims(heads)
        q_np, cache_np = _inputs(seed, heads, n_rows, rows)
        q, cache, r = _dev(dev, q_np, cache_np, rows)
        got = _noalloc_result(dims, q, cache, r)
        ref = _workspace_result(dims, q, cache, r)
        torch.cuda.synchronize()
        assert not torch.isnan(got[1]).any()   # no wait gave up (the combine would write NaN)
        _check(q_np, cache_np, rows, got, ref)


def test_noalloc_refuses_requests_beyond_its_scratch():
    dev = torch.device("cuda:0")
    dims = kp.make_dims(128)
    q = torch.zeros(8, 128, 512, dtype=torch.bfloat16, device=dev)       # 8 x 1024 x 128 partials
    cache = torch.zeros(64, 528, dtype=torch.int8, device=dev)
    rows = torch.full((8, 65536), -1, dtype=torch.int32, device=dev)
    out = torch.empty(8, 128, 512, dtype=torch.bfloat16, device=dev)
    with pytest.raises(kp.GlmError) as e:
        kp.glm_sparse_mla_decode_noalloc(dims, q, cache, rows, 0.04, out)
    assert e.value.status == kp.GLM_ERR_WORKSPACE
