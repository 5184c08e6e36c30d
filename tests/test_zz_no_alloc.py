"""The allocation-free sparse MLA entry point (glm_sparse_mla_decode_noalloc).

It serves callers that cannot allocate device memory where they run the attention (plugin
interfaces that pass only inputs and outputs; serving loops that allow no allocation after
start-up). Its split partials live in a fixed scratch array inside the library instead of a
caller workspace. Through the C ABI, two calls in a row -- with different shapes, so that stale
scratch from the first call would show -- must give the results of the workspace entry point
glm_sparse_mla_decode within the attention tolerance of the parity tests, and a request larger
than the scratch must be refused. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp
import oracle
import synth

pytestmark = pytest.mark.gpu


def _case(dev, seed, n_heads, n_q, width, n_valid, n_rows):
    rng = np.random.default_rng(seed)
    lat = synth.f32_to_bf16_bits(rng.standard_normal((n_rows, 512)).astype(np.float32))
    cache = np.zeros((n_rows, 528), np.int8)
    oracle.store_int8(lat, np.arange(n_rows, dtype=np.int64), cache)   # inputs only
    rows = np.full((n_q, width), -1, np.int32)
    for n in range(n_q):
        rows[n, :n_valid] = rng.choice(n_rows, size=n_valid, replace=False)
    q = synth.f32_to_bf16_bits(rng.standard_normal((n_q, n_heads, 512)).astype(np.float32))
    t = lambda a, dt: torch.from_numpy(a).to(dev) if dt is None else torch.from_numpy(a.view(np.int16)).view(dt).to(dev)  # noqa: E731
    return t(q, torch.bfloat16), t(cache, None), t(rows, None)


def _workspace_result(dims, q, cache, rows, sm):
    n_q, heads = q.shape[0], q.shape[1]
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, n_q, width=rows.shape[1]),
                     dtype=torch.uint8, device=q.device)
    out = torch.empty(n_q, heads, 512, dtype=torch.bfloat16, device=q.device)
    o32 = torch.empty(n_q, heads, 512, dtype=torch.float32, device=q.device)
    lse = torch.empty(n_q, heads, dtype=torch.float32, device=q.device)
    kp.glm_sparse_mla_decode(dims, q, cache, rows, sm, out, ws, lse=lse, out_f32=o32)
    return out, o32, lse


def _noalloc_result(dims, q, cache, rows, sm):
    n_q, heads = q.shape[0], q.shape[1]
    out = torch.full((n_q, heads, 512), 9.0, dtype=torch.bfloat16, device=q.device)
    o32 = torch.full((n_q, heads, 512), 9.0, dtype=torch.float32, device=q.device)
    lse = torch.full((n_q, heads), 9.0, dtype=torch.float32, device=q.device)
    kp.glm_sparse_mla_decode_noalloc(dims, q, cache, rows, sm, out, lse=lse, out_f32=o32)
    return out, o32, lse


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    max_abs = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert max_abs <= 1e-2 and rel <= 5e-3, (max_abs, rel)


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    dev = torch.device("cuda:0")
    sm = float(np.float32(512 ** -0.5))
    cases = [dict(seed=1, n_heads=64, n_q=2, width=2176, n_valid=2048, n_rows=6000),
             dict(seed=2, n_heads=16, n_q=3, width=80, n_valid=67, n_rows=500)]
    for c in cases:
        dims = kp.make_dims(c["n_heads"])
        q, cache, rows = _case(dev, c["seed"], c["n_heads"], c["n_q"], c["width"], c["n_valid"], c["n_rows"])
        ref = _workspace_result(dims, q, cache, rows, sm)
        got = _noalloc_result(dims, q, cache, rows, sm)
        torch.cuda.synchronize()
        _close(got[1], ref[1])                                   # fp32 output
        _close(got[0].float(), ref[0].float())                   # bf16 output
        np.testing.assert_allclose(got[2].cpu().numpy(), ref[2].cpu().numpy(), atol=1e-3, rtol=0)


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
