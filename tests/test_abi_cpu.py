"""The C-ABI library loads, exports every function include/glm_dsa.h declares, and rejects bad
arguments on the host before any CUDA call (so these run without a GPU)."""
import ctypes as C
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT

kp = pytest.importorskip("kpool_indexer_int8_b200")


def _declared():
    src = open(os.path.join(ROOT, "include", "glm_dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(glm_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(kp.lib, n), n
    assert set(kp.EXPORTS) <= set(names)


def test_dims_check_nope_and_geometry():
    ok = kp.make_dims(64)
    assert kp.check_dims(ok) == kp.GLM_OK
    assert kp.check_dims(kp.make_dims(64, qk_rope_head_dim=64)) == kp.GLM_ERR_UNSUPPORTED
    assert kp.check_dims(kp.make_dims(64, kv_lora_rank=576)) == kp.GLM_ERR_UNSUPPORTED
    assert kp.check_dims(kp.make_dims(64, index_kpool=8)) == kp.GLM_ERR_UNSUPPORTED
    assert kp.check_dims(kp.make_dims(0)) == kp.GLM_ERR_UNSUPPORTED
    assert kp.check_dims(kp.make_dims(129)) == kp.GLM_ERR_UNSUPPORTED
    assert kp.check_dims(kp.make_dims(16, index_topk=2047)) == kp.GLM_ERR_INVALID_ARG
    assert kp.lib.glm_check_dims(None) == kp.GLM_ERR_INVALID_ARG
    assert kp.lib.glm_status_string(kp.GLM_ERR_WORKSPACE) == b"workspace missing or too small"


def test_workspace_sizes():
    d = kp.make_dims(64)
    assert kp.glm_dsa_workspace_size(d, kp.GLM_OP_INDEX_SCORES_TOPK, 1, 65536, 512) >= 65536 * 4
    mla = kp.glm_dsa_workspace_size(d, kp.GLM_OP_SPARSE_MLA, 1, width=2176)
    assert mla >= 2176 // 64 * 64 * 512 * 4
    assert kp.glm_dsa_workspace_size(d, kp.GLM_OP_SPARSE_MLA, 2, width=2176) >= 2 * mla - 512
    with pytest.raises(kp.GlmError):
        kp.glm_dsa_workspace_size(d, kp.GLM_OP_INDEX_SCORES_TOPK, 1, 100, 4096)
    with pytest.raises(kp.GlmError):
        kp.glm_dsa_workspace_size(d, 99, 1)
    with pytest.raises(kp.GlmError):
        kp.glm_dsa_workspace_size(kp.make_dims(64, qk_rope_head_dim=64), kp.GLM_OP_SPARSE_MLA, 1, width=8)


FAKE = C.c_void_p(0x10000)        # 16-byte aligned, never dereferenced: every call below fails first
MIS = C.c_void_p(0x10004)         # misaligned for 16-byte operands


def test_workspace_sizes_cover_every_smaller_query_count():
    # a workspace sized for n_q queries serves any smaller count: the attention's plan changes
    # with the count (one partial per chunk for few queries, runs of chunks for many), the size
    # must not shrink as the count grows; the many-query index scratch likewise
    for heads in (16, 64, 128):
        d = kp.make_dims(heads)
        for op, kw in ((kp.GLM_OP_SPARSE_MLA, dict(width=2176)),
                       (kp.GLM_OP_INDEX_SCORES_TOPK, dict(max_pools=33792, select_k=512)),
                       (kp.GLM_OP_DECODE_STEP, dict(max_pools=33792, select_k=512, width=2176))):
            prev = 0
            for nq in sorted(set(range(1, 400, 7)) | {127, 128, 129, 295, 296, 297, 591, 592, 593, 1000, 4096, 65535}):
                size = kp.glm_dsa_workspace_size(d, op, nq, **kw)
                assert size >= prev, (heads, op, nq)
                prev = size


def test_step_plan_counts_the_kernels_of_each_path():
    d = kp.make_dims(64)
    # one decode query: step_prep, the fused index kernel, the split attention and its combine
    assert kp.glm_dsa_step_plan(d, 1, 65536, 1, 2176) == (4, kp.GLM_PLAN_MLA_COMBINE)
    # 4,096 prefill queries: step_prep, query preparation, scores, histogram, selection, expansion,
    # the walking attention writing its output (one run per query)
    k, f = kp.glm_dsa_step_plan(d, 4096, 33792, 1, 2176)
    assert (k, f) == (7, kp.GLM_PLAN_INDEX_MANY | kp.GLM_PLAN_MLA_MANY)
    # the INT8 indexer state keeps the fused index kernel
    assert kp.glm_dsa_step_plan(d, 4096, 33792, 1, 2176, int8_keys=True)[1] == kp.GLM_PLAN_MLA_MANY
    # no query: step_prep only
    assert kp.glm_dsa_step_plan(d, 0, 16, 1, 2176) == (1, 0)
    with pytest.raises(kp.GlmError):
        kp.glm_dsa_step_plan(d, -1, 16, 1, 2176)


def test_store_rejects_before_launch():
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    bad = C.byref(kp.make_dims(64, qk_rope_head_dim=64))
    assert L.glm_kv_store_int8(bad, FAKE, FAKE, 1, FAKE, 1, None) == kp.GLM_ERR_UNSUPPORTED
    assert L.glm_kv_store_int8(d, FAKE, FAKE, -1, FAKE, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_int8(d, None, FAKE, 1, FAKE, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_int8(d, MIS, FAKE, 1, FAKE, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_int8(d, FAKE, FAKE, 1, MIS, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_int8(d, None, None, 0, None, 0, None) == kp.GLM_OK   # n == 0: no-op


def test_expand_requires_room_for_selection_and_tail():
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    # out_width must be >= 4 * select_k + 3
    assert L.glm_expand_selection(d, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 1, 512, None, 0, 2050,
                                  FAKE, None, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_expand_selection(d, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 0, 512, None, 0, 2051,
                                  FAKE, None, None) == kp.GLM_OK          # n_q == 0: no-op
    assert L.glm_expand_selection(d, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 1, 512, None, 0, 2051,
                                  None, None, None) == kp.GLM_ERR_INVALID_ARG  # no output


def test_fused_index_expand_argument_checks():
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    args = lambda sk, ow, tok, rows, ws_bytes: (d, FAKE, FAKE, FAKE, 16, FAKE, FAKE, FAKE, FAKE, 1, 1, sk,  # noqa: E731
                                                None, 0, ow, None, FAKE, None, tok, rows, FAKE, ws_bytes, None)
    # out_width must hold the largest selection plus a full tail
    assert L.glm_index_topk_expand(*args(512, 2050, FAKE, None, 1 << 30)) == kp.GLM_ERR_INVALID_ARG
    # no expansion output at all
    assert L.glm_index_topk_expand(*args(512, 2051, None, None, 1 << 30)) == kp.GLM_ERR_INVALID_ARG
    # misaligned expansion output
    assert L.glm_index_topk_expand(*args(512, 2051, C.c_void_p(0x10002), None, 1 << 30)) == kp.GLM_ERR_INVALID_ARG
    # select_k out of range, then a workspace that is too small
    assert L.glm_index_topk_expand(*args(4096, 16387, FAKE, None, 1 << 30)) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_index_topk_expand(*args(8, 35, FAKE, FAKE, 16)) == kp.GLM_ERR_WORKSPACE


def test_index_and_mla_argument_checks():
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    # select_k out of range
    assert L.glm_index_scores_topk(d, FAKE, FAKE, FAKE, 16, FAKE, FAKE, FAKE, FAKE, 1, 1, 4096, None,
                                   FAKE, None, FAKE, 1 << 20, None) == kp.GLM_ERR_INVALID_ARG
    # missing workspace when scores are not given
    assert L.glm_index_scores_topk(d, FAKE, FAKE, FAKE, 16, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, None,
                                   FAKE, None, None, 0, None) == kp.GLM_ERR_WORKSPACE
    # MLA: workspace too small, width out of range, misaligned q
    assert L.glm_sparse_mla_decode(d, FAKE, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE, 16,
                                   None) == kp.GLM_ERR_WORKSPACE
    assert L.glm_sparse_mla_decode(d, FAKE, FAKE, 10, FAKE, 1, 0, 0.04, FAKE, None, None, FAKE, 1 << 30,
                                   None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_sparse_mla_decode(d, MIS, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE, 1 << 30,
                                   None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_topk_pools(FAKE, 16, FAKE, 1, 0, FAKE, None, None, 0, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kpool_build(d, FAKE, FAKE, 16, FAKE, FAKE, C.c_float(-1.0), FAKE, FAKE, None, 1, 1,
                             FAKE, 4, None, None) == kp.GLM_ERR_INVALID_ARG


def test_step_struct_layout_matches_the_header(tmp_path):
    # the ctypes mirror of glm_dsa_step must have the C compiler's field offsets and size
    fields = [f for f, _ in kp.glm_dsa_step._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "glm_dsa.h"\nint main(void) {\n' +
                   "".join(f'    printf("%zu\\n", offsetof(glm_dsa_step, {f}));\n' for f in fields) +
                   '    printf("%zu\\n", sizeof(glm_dsa_step));\n    return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    want = [getattr(kp.glm_dsa_step, f).offset for f in fields] + [C.sizeof(kp.glm_dsa_step)]
    assert got == want


def test_step_argument_checks():
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    assert L.glm_dsa_decode_step(d, None, FAKE, 1 << 30, None) == kp.GLM_ERR_INVALID_ARG
    a = kp.glm_dsa_step()                       # all counts zero, every pointer NULL
    a.out_width, a.select_k, a.sm_scale = 2051, 512, 0.04
    a.ld_pools = 16
    assert L.glm_dsa_decode_step(d, C.byref(a), None, 0, None) == kp.GLM_ERR_WORKSPACE    # nothing else missing
    a.out_width = 2050                         # below 4 * select_k + 3
    assert L.glm_dsa_decode_step(d, C.byref(a), FAKE, 1 << 30, None) == kp.GLM_ERR_INVALID_ARG
    a.out_width = 2051
    a.n_new, a.latent_dev = 1, None             # a new row without its latent
    assert L.glm_dsa_decode_step(d, C.byref(a), FAKE, 1 << 30, None) == kp.GLM_ERR_INVALID_ARG
    a.n_new = 0
    need = kp.glm_dsa_workspace_size(kp.make_dims(64), kp.GLM_OP_DECODE_STEP, 0, 16, 512, 2051)
    assert L.glm_dsa_decode_step(d, C.byref(a), FAKE, need - 1, None) == kp.GLM_ERR_WORKSPACE


def test_fp8_entry_points_reject_before_launch():
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    bad = C.byref(kp.make_dims(64, qk_rope_head_dim=64))
    assert L.glm_kv_store_fp8(bad, FAKE, FAKE, 1, FAKE, 1, None) == kp.GLM_ERR_UNSUPPORTED
    assert L.glm_kv_store_fp8(d, None, FAKE, 1, FAKE, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_fp8(d, FAKE, FAKE, 1, MIS, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_fp8(d, None, None, 0, None, 0, None) == kp.GLM_OK        # n == 0: no-op
    assert L.glm_sparse_mla_decode_fp8(bad, FAKE, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE,
                                       1 << 30, None) == kp.GLM_ERR_UNSUPPORTED
    assert L.glm_sparse_mla_decode_fp8(d, FAKE, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE, 16,
                                       None) == kp.GLM_ERR_WORKSPACE
    assert L.glm_sparse_mla_decode_fp8(d, FAKE, FAKE, 10, FAKE, 1, 0, 0.04, FAKE, None, None, FAKE,
                                       1 << 30, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_sparse_mla_decode_fp8(d, MIS, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE,
                                       1 << 30, None) == kp.GLM_ERR_INVALID_ARG


def test_fp4_entry_points_reject_before_launch():
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    bad = C.byref(kp.make_dims(64, qk_rope_head_dim=64))
    assert L.glm_kv_store_fp4(bad, FAKE, FAKE, 1, FAKE, 1, None) == kp.GLM_ERR_UNSUPPORTED
    assert L.glm_kv_store_fp4(d, None, FAKE, 1, FAKE, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_fp4(d, FAKE, FAKE, 1, MIS, 1, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_kv_store_fp4(d, None, None, 0, None, 0, None) == kp.GLM_OK        # n == 0: no-op
    assert L.glm_sparse_mla_decode_fp4(bad, FAKE, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE,
                                       1 << 30, None) == kp.GLM_ERR_UNSUPPORTED
    assert L.glm_sparse_mla_decode_fp4(d, FAKE, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE, 16,
                                       None) == kp.GLM_ERR_WORKSPACE
    assert L.glm_sparse_mla_decode_fp4(d, FAKE, MIS, 10, FAKE, 1, 64, 0.04, FAKE, None, None, FAKE,
                                       1 << 30, None) == kp.GLM_ERR_INVALID_ARG
    # a cache format other than int8, fp8 and fp4 is rejected before anything else is looked at
    a = kp.glm_dsa_step()
    for fmt in (-1, 3):
        a.cache_format = fmt
        assert L.glm_dsa_decode_step(d, C.byref(a), FAKE, 1 << 30, None) == kp.GLM_ERR_INVALID_ARG


def test_noalloc_entry_rejects_before_launch():
    # the allocation-free MLA entry point runs the workspace entry's checks: every rejection below
    # happens on the host, before its scratch is looked up or anything is enqueued
    L = kp.lib
    d = C.byref(kp.make_dims(64))
    bad = C.byref(kp.make_dims(64, qk_rope_head_dim=64))
    assert L.glm_sparse_mla_decode_noalloc(bad, FAKE, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None,
                                           None) == kp.GLM_ERR_UNSUPPORTED
    assert L.glm_sparse_mla_decode_noalloc(d, FAKE, FAKE, 10, FAKE, 1, 0, 0.04, FAKE, None, None,
                                           None) == kp.GLM_ERR_INVALID_ARG        # width 0
    assert L.glm_sparse_mla_decode_noalloc(d, FAKE, FAKE, 10, FAKE, -1, 64, 0.04, FAKE, None, None,
                                           None) == kp.GLM_ERR_INVALID_ARG        # n_q < 0
    assert L.glm_sparse_mla_decode_noalloc(d, None, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None,
                                           None) == kp.GLM_ERR_INVALID_ARG        # null q
    assert L.glm_sparse_mla_decode_noalloc(d, FAKE, FAKE, 10, None, 1, 64, 0.04, FAKE, None, None,
                                           None) == kp.GLM_ERR_INVALID_ARG        # null rows
    assert L.glm_sparse_mla_decode_noalloc(d, MIS, FAKE, 10, FAKE, 1, 64, 0.04, FAKE, None, None,
                                           None) == kp.GLM_ERR_INVALID_ARG        # misaligned q
    assert L.glm_sparse_mla_decode_noalloc(d, FAKE, FAKE, 10, FAKE, 1, 64, C.c_float(float("nan")), FAKE,
                                           None, None, None) == kp.GLM_ERR_INVALID_ARG
    assert L.glm_sparse_mla_decode_noalloc(d, None, None, 0, None, 0, 64, 0.04, None, None, None,
                                           None) == kp.GLM_OK                     # n_q == 0: no-op
    # more partials than the scratch holds: refused before any CUDA call
    d128 = C.byref(kp.make_dims(128))
    assert L.glm_sparse_mla_decode_noalloc(d128, FAKE, FAKE, 10, FAKE, 8, 65536, 0.04, FAKE, None, None,
                                           None) == kp.GLM_ERR_WORKSPACE


def test_algorithmic_bytes_of_the_tiny_decode():
    # by hand: 128 visible pools x 512 B + q_idx 8,192 B + w 128 B + 16 top-k ids x 4 B; 64 gathered
    # rows x 528 B + q and out 2 x 16 heads x 1,024 B + 80 indices x 4 B; one new row (1,024 B in,
    # 528 B out, 8 B slot); one completed pool (4 x 512 B of k and gate in, 512 B out)
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import synth
    ab = bench.algorithmic_bytes(synth.generate(synth.TINY_DECODE))
    assert ab["index"] == 128 * 512 + 8192 + 128 + 16 * 4
    assert ab["mla"] == 64 * 528 + 2 * 16 * 1024 + 80 * 4
    assert ab["store"] == 1560 and ab["kpool"] == 2560 and ab["gathered"] == 64
    assert ab["total"] == ab["index"] + ab["mla"] + ab["store"] + ab["kpool"] == 144920


def test_algorithmic_bytes_count_a_prefill_chunks_shared_data_once():
    # 300 causal queries at the end of one 6,000-token sequence: its 1,500 pooled keys once (the
    # last query sees them all) and its rows at most once each (the queries gather 300 x 512 and
    # more of them); per query q_idx + w + 128 top-k ids, q + out (64 heads) + 515 indices
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import synth
    wl = synth.custom("prefill_bytes", (0,), (6000,), n_heads=64, select_k=128, out_width=515, chunk=300, seed=44)
    ab = bench.algorithmic_bytes(synth.generate(wl))
    assert ab["index"] == 1500 * 512 + 300 * (8192 + 128 + 128 * 4)
    assert ab["mla"] == 6000 * 528 + 300 * (2 * 64 * 1024 + 515 * 4)
    assert ab["gathered"] >= 300 * 512   # the attention's work stays per (query, row)


def test_bench_stage_names_follow_the_step_plan():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import synth
    k, paths, names = bench.step_kernels(kp, synth.WORKLOADS["long_decode"], 65536, False)
    assert k == 4 and names == ("step_prep", "index_select_tc", "mla_split_tc", "mla_combine")
    k, paths, names = bench.step_kernels(kp, synth.CHUNKED_PREFILL, 33792, False)
    assert k == 7 and paths == kp.GLM_PLAN_INDEX_MANY | kp.GLM_PLAN_MLA_MANY
    assert "index_gemm" in names[1] and names[2] == "mla_multi_tc" and "no combine" in names[3]
