"""fp64 CPU oracle of the GLM-5.3-Flash kpool DSA decode path (numpy front end of oracle.c).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package. It shares no code with the CUDA path
(``kpool_indexer_int8_b200``) and does not import it; inputs come from ``synth``.

The arithmetic lives in ``oracle.c`` (plain single-threaded C, fp64); this module only marshals
numpy arrays and composes the steps in the order the pages give them ("Module glm5next_dsa_ref":
pool_states -> index_scores -> topk_pools -> expand_selection -> mla_masked_attention;
"GLM-5.3 Kernels": store_int8 -> sparse MLA over the gathered rows).
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

ROW_BYTES = 528
LATENT = 512
KPOOL = 4
INVALID = -1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = C.CDLL(path)
        _declare(_lib)
    return _lib


_p = C.c_void_p
_i64 = C.c_int64
_i32 = C.c_int
_f64 = C.c_double


def _declare(L):
    L.oracle_check_dims.argtypes = [_i32] * 6
    L.oracle_check_dims.restype = _i32
    L.oracle_store_int8.argtypes = [_p, _p, _i64, _p, _i64]
    L.oracle_store_int8.restype = _i32
    L.oracle_dequant_row.argtypes = [_p, _i64, _p]
    L.oracle_dequant_row.restype = None
    L.oracle_layer_norm.argtypes = [_p, _i32, _p, _p, _f64, _p]
    L.oracle_layer_norm.restype = None
    L.oracle_visible.argtypes = [_i64, _i64, _i64, _i64]
    L.oracle_visible.restype = _i32
    L.oracle_n_pools.argtypes = [_i64, _i32]
    L.oracle_n_pools.restype = _i64
    L.oracle_n_visible_pools.argtypes = [_i64, _i64, _i64, _i32]
    L.oracle_n_visible_pools.restype = _i64
    L.oracle_pool_states.argtypes = [_p, _p, _i32, _i64, _i64, _i32, _p, _p, _f64, _p]
    L.oracle_pool_states.restype = _i64
    L.oracle_index_scores.argtypes = [_p, _p, _p, _i32, _i32, _i64, _p]
    L.oracle_index_scores.restype = None
    L.oracle_pool_q8.argtypes = [_p, _i32, _p, _p]
    L.oracle_pool_q8.restype = None
    L.oracle_index_scores_q8.argtypes = [_p, _p, _p, _p, _i32, _i32, _i64, _p]
    L.oracle_index_scores_q8.restype = None
    L.oracle_topk_pools.argtypes = [_p, _i64, _i64, _p]
    L.oracle_topk_pools.restype = _i64
    L.oracle_expand_selection.argtypes = [_p, _i64, _i64, _i64, _i64, _i32, _i64, _p]
    L.oracle_expand_selection.restype = _i64
    L.oracle_rows_from_tokens.argtypes = [_p, _i64, _p, _p]
    L.oracle_rows_from_tokens.restype = None
    L.oracle_sparse_mla.argtypes = [_p, _i32, _p, _i64, _p, _i64, _f64, _p, _p]
    L.oracle_sparse_mla.restype = _i32
    L.oracle_topk_to_mask.argtypes = [_p, _i64, _i64, _p]
    L.oracle_topk_to_mask.restype = None
    L.oracle_masked_attention.argtypes = [_p, _i32, _p, _i64, _p, _i64, _p, _f64, _p, _p]
    L.oracle_masked_attention.restype = _i32
    L.oracle_expand_kv.argtypes = [_p, _i64, _i32, _p, _i32, _i32, _i32, _p, _p]
    L.oracle_expand_kv.restype = None
    L.oracle_q_absorb.argtypes = [_p, _i32, _i32, _p, _i32, _i32, _p]
    L.oracle_q_absorb.restype = None
    L.oracle_v_up.argtypes = [_p, _i32, _i32, _p, _i32, _i32, _p]
    L.oracle_v_up.restype = None
    L.oracle_attention_f64.argtypes = [_p, _i32, _i32, _p, _p, _i64, _i32, _i32, _f64, _p]
    L.oracle_attention_f64.restype = None
    L.oracle_e4m3_value.argtypes = [C.c_uint]
    L.oracle_e4m3_value.restype = _f64
    L.oracle_e4m3_encode.argtypes = [_f64]
    L.oracle_e4m3_encode.restype = C.c_uint
    L.oracle_store_fp8.argtypes = [_p, _p, _i64, _p, _i64]
    L.oracle_store_fp8.restype = _i32
    L.oracle_dequant_row_fp8.argtypes = [_p, _i64, _p]
    L.oracle_dequant_row_fp8.restype = None
    L.oracle_e2m1_value.argtypes = [C.c_uint]
    L.oracle_e2m1_value.restype = _f64
    L.oracle_e2m1_encode.argtypes = [_f64]
    L.oracle_e2m1_encode.restype = C.c_uint
    L.oracle_store_fp4.argtypes = [_p, _p, _i64, _p, _i64]
    L.oracle_store_fp4.restype = _i32
    L.oracle_dequant_row_fp4.argtypes = [_p, _i64, _p]
    L.oracle_dequant_row_fp4.restype = None


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(C.c_void_p)


# ------------------------------------------------------------------------------------------------
# one function per oracle step
# ------------------------------------------------------------------------------------------------

def check_dims(kv_lora_rank=512, qk_rope_head_dim=0, n_heads=64, index_n_heads=32,
               index_head_dim=128, index_kpool=4) -> bool:
    return lib().oracle_check_dims(kv_lora_rank, qk_rope_head_dim, n_heads, index_n_heads,
                                   index_head_dim, index_kpool) == 0


def store_int8(latent, slots, cache) -> None:
    """Quantise ``latent`` (uint16 bf16 bits [n, 512]) into ``cache`` (int8 [n_rows, 528]) in place."""
    assert cache.dtype == np.int8 and cache.flags.c_contiguous and cache.shape[-1] == ROW_BYTES
    lat, lp = _c(latent, np.uint16)
    sl, sp = _c(slots, np.int64)
    assert lat.shape == (sl.shape[0], LATENT)
    rc = lib().oracle_store_int8(lp, sp, sl.shape[0], cache.ctypes.data_as(C.c_void_p),
                                 cache.reshape(-1, ROW_BYTES).shape[0])
    if rc != 0:
        raise ValueError("slot past the end of the cache")


def dequant_rows(cache, rows) -> np.ndarray:
    cache = np.ascontiguousarray(cache, dtype=np.int8).reshape(-1, ROW_BYTES)
    out = np.empty((len(rows), LATENT), dtype=np.float64)
    for i, r in enumerate(rows):
        lib().oracle_dequant_row(cache.ctypes.data_as(C.c_void_p), int(r),
                                 out[i].ctypes.data_as(C.c_void_p))
    return out


def layer_norm(x, w, b, eps) -> np.ndarray:
    x, xp = _c(x, np.float64)
    w, wp = _c(w, np.float64)
    b, bp = _c(b, np.float64)
    y = np.empty_like(x)
    lib().oracle_layer_norm(xp, x.shape[0], wp, bp, float(eps), y.ctypes.data_as(C.c_void_p))
    return y


def visible(pad, length, q_pos, t) -> bool:
    return bool(lib().oracle_visible(int(pad), int(length), int(q_pos), int(t)))


def n_pools(length, kpool=KPOOL) -> int:
    return int(lib().oracle_n_pools(int(length), kpool))


def n_visible_pools(pad, length, q_pos, kpool=KPOOL) -> int:
    return int(lib().oracle_n_visible_pools(int(pad), int(length), int(q_pos), kpool))


def pool_states(k_seq, gate_seq, pad, length, ln_w, ln_b, eps, kpool=KPOOL) -> np.ndarray:
    """Pools of one sequence. ``k_seq``/``gate_seq``: uint16 bf16 bits [>= pad+len, d] in padded
    coordinates. Returns float64 [len // kpool, d]."""
    k, kp = _c(k_seq, np.uint16)
    g, gp = _c(gate_seq, np.uint16)
    d = k.shape[1]
    assert k.shape[0] >= pad + length and g.shape == k.shape
    w, wp = _c(ln_w, np.float32)
    b, bp = _c(ln_b, np.float32)
    out = np.empty((max(n_pools(length, kpool), 0), d), dtype=np.float64)
    n = lib().oracle_pool_states(kp, gp, d, int(pad), int(length), kpool, wp, bp, float(eps),
                                 out.ctypes.data_as(C.c_void_p))
    assert n == out.shape[0]
    return out


def index_scores(q_idx, w, pooled, n_vis) -> np.ndarray:
    """``q_idx`` uint16 bf16 bits [H, D]; ``w`` float32 [H]; ``pooled`` [P, D] (any float dtype,
    widened exactly to fp64). Returns float64 [n_vis]."""
    q, qp = _c(q_idx, np.uint16)
    w, wp = _c(w, np.float32)
    pl, pp = _c(pooled, np.float64)
    H, D = q.shape
    assert pl.shape[1] == D and pl.shape[0] >= n_vis and w.shape == (H,)
    out = np.empty(int(n_vis), dtype=np.float64)
    lib().oracle_index_scores(qp, wp, pp, H, D, int(n_vis), out.ctypes.data_as(C.c_void_p))
    return out


def pool_q8(pooled32):
    """INT8 indexer state of fp32 pooled keys ``pooled32`` [P, D] (float32): returns
    (codes int8 [P, D], scales float32 [P]), one scale per row."""
    x = np.ascontiguousarray(pooled32, dtype=np.float32)
    P, D = x.shape
    codes = np.empty((P, D), dtype=np.int8)
    scales = np.empty(P, dtype=np.float32)
    for p in range(P):
        lib().oracle_pool_q8(x[p].ctypes.data_as(C.c_void_p), D, codes[p].ctypes.data_as(C.c_void_p),
                             scales[p:].ctypes.data_as(C.c_void_p))
    return codes, scales


def index_scores_q8(q_idx, w, codes, scales, n_vis) -> np.ndarray:
    """Scores on the INT8 indexer state: ``codes`` int8 [P, D], ``scales`` float32 [P]."""
    q, qp = _c(q_idx, np.uint16)
    w, wp = _c(w, np.float32)
    c, cp = _c(codes, np.int8)
    sc, sp = _c(scales, np.float32)
    H, D = q.shape
    assert c.shape[1] == D and c.shape[0] >= n_vis and sc.shape[0] >= n_vis and w.shape == (H,)
    out = np.empty(int(n_vis), dtype=np.float64)
    lib().oracle_index_scores_q8(qp, wp, cp, sp, H, D, int(n_vis), out.ctypes.data_as(C.c_void_p))
    return out


def topk_pools(scores, select_k):
    s, sp = _c(scores, np.float64)
    out = np.empty(int(select_k), dtype=np.int32)
    n_sel = lib().oracle_topk_pools(sp, s.shape[0], int(select_k), out.ctypes.data_as(C.c_void_p))
    return out, int(n_sel)


def expand_selection(topk, n_sel, pad, length, q_pos, out_width, kpool=KPOOL):
    t, tp = _c(topk, np.int32)
    out = np.empty(int(out_width), dtype=np.int32)
    n = lib().oracle_expand_selection(tp, int(n_sel), int(pad), int(length), int(q_pos), kpool,
                                      int(out_width), out.ctypes.data_as(C.c_void_p))
    if n < 0:
        raise ValueError("selection does not fit in out_width")
    return out, int(n)


def rows_from_tokens(tok, slot_map_row) -> np.ndarray:
    t, tp = _c(tok, np.int32)
    m, mp = _c(slot_map_row, np.int64)
    out = np.empty_like(t)
    lib().oracle_rows_from_tokens(tp, t.shape[0], mp, out.ctypes.data_as(C.c_void_p))
    return out


def sparse_mla(q, cache, rows, sm_scale):
    """``q`` uint16 bf16 bits [Hm, 512]; ``cache`` int8 [n_rows, 528]; ``rows`` int32 [W].
    Returns (out float64 [Hm, 512], lse float64 [Hm])."""
    qq, qp = _c(q, np.uint16)
    cache = np.ascontiguousarray(cache, dtype=np.int8).reshape(-1, ROW_BYTES)
    r, rp = _c(rows, np.int32)
    Hm = qq.shape[0]
    out = np.empty((Hm, LATENT), dtype=np.float64)
    lse = np.empty(Hm, dtype=np.float64)
    rc = lib().oracle_sparse_mla(qp, Hm, cache.ctypes.data_as(C.c_void_p), cache.shape[0], rp,
                                 r.shape[0], float(sm_scale), out.ctypes.data_as(C.c_void_p),
                                 lse.ctypes.data_as(C.c_void_p))
    if rc != 0:
        raise ValueError("index past the end of the cache")
    return out, lse


def topk_to_mask(tok, n_tok) -> np.ndarray:
    t, tp = _c(tok, np.int32)
    mask = np.empty(int(n_tok), dtype=np.uint8)
    lib().oracle_topk_to_mask(tp, t.shape[0], int(n_tok), mask.ctypes.data_as(C.c_void_p))
    return mask.astype(bool)


def masked_attention(q, cache, slot_map_row, mask, sm_scale):
    qq, qp = _c(q, np.uint16)
    cache = np.ascontiguousarray(cache, dtype=np.int8).reshape(-1, ROW_BYTES)
    sm, smp = _c(slot_map_row, np.int64)
    mk, mkp = _c(mask, np.uint8)
    Hm = qq.shape[0]
    out = np.empty((Hm, LATENT), dtype=np.float64)
    lse = np.empty(Hm, dtype=np.float64)
    rc = lib().oracle_masked_attention(qp, Hm, cache.ctypes.data_as(C.c_void_p), cache.shape[0],
                                       smp, mk.shape[0], mkp, float(sm_scale),
                                       out.ctypes.data_as(C.c_void_p),
                                       lse.ctypes.data_as(C.c_void_p))
    if rc != 0:
        raise ValueError("index past the end of the cache")
    return out, lse


# ------------------------------------------------------------------------------------------------
# the MLA up-projection ("Module glm5next_dsa_ref", expand_kv; kv_b_proj rows grouped per head,
# the dk K rows of a head, then its dv V rows; weights as bf16 bits [Hm * (dk + dv), L])
# ------------------------------------------------------------------------------------------------

def _as_f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(C.c_void_p)


def expand_kv(c, w_kv_b, n_heads, dk, dv):
    """Per-head K [Hm, T, dk] and V [Hm, T, dv] of latent rows ``c`` float64 [T, L]."""
    cc, cp = _as_f64(c)
    w, wp = _c(w_kv_b, np.uint16)
    T, L = cc.shape
    k = np.empty((n_heads, T, dk), dtype=np.float64)
    v = np.empty((n_heads, T, dv), dtype=np.float64)
    lib().oracle_expand_kv(cp, T, L, wp, n_heads, dk, dv, k.ctypes.data_as(C.c_void_p),
                           v.ctypes.data_as(C.c_void_p))
    return k, v


def q_absorb(q, w_kv_b, dk, dv, latent=LATENT):
    """Latent-space queries [Hm, L] of per-head queries ``q`` float64 [Hm, dk]."""
    qq, qp = _as_f64(q)
    w, wp = _c(w_kv_b, np.uint16)
    out = np.empty((qq.shape[0], latent), dtype=np.float64)
    lib().oracle_q_absorb(qp, qq.shape[0], latent, wp, dk, dv, out.ctypes.data_as(C.c_void_p))
    return out


def v_up(o_lat, w_kv_b, dk, dv):
    """The up-projection of latent-space outputs ``o_lat`` float64 [Hm, L] to [Hm, dv]."""
    oo, op = _as_f64(o_lat)
    w, wp = _c(w_kv_b, np.uint16)
    out = np.empty((oo.shape[0], dv), dtype=np.float64)
    lib().oracle_v_up(op, oo.shape[0], oo.shape[1], wp, dk, dv, out.ctypes.data_as(C.c_void_p))
    return out


def attention_f64(q, k, v, scale, shared):
    """Softmax attention in fp64: ``q`` [Hm, dq]; ``k`` [Hm, T, dq] and ``v`` [Hm, T, dv] per head,
    or [T, dq] and [T, dv] for every head when ``shared``. Returns [Hm, dv]."""
    qq, qp = _as_f64(q)
    kk, kp = _as_f64(k)
    vv, vp = _as_f64(v)
    T = kk.shape[-2]
    out = np.empty((qq.shape[0], vv.shape[-1]), dtype=np.float64)
    lib().oracle_attention_f64(qp, qq.shape[0], qq.shape[1], kp, vp, T, vv.shape[-1], 1 if shared else 0,
                               float(scale), out.ctypes.data_as(C.c_void_p))
    return out


# ------------------------------------------------------------------------------------------------
# the FP8 latent cache row (E4M3 codes, one fp32 scale per row, the INT8 row's 528-byte layout)
# ------------------------------------------------------------------------------------------------

def e4m3_value(code) -> float:
    return lib().oracle_e4m3_value(int(code) & 0xFF)


def e4m3_encode(x) -> int:
    return int(lib().oracle_e4m3_encode(float(x)))


def store_fp8(latent, slots, cache) -> None:
    """Quantise ``latent`` (uint16 bf16 bits [n, 512]) into ``cache`` (uint8 [n_rows, 528]) in place."""
    assert cache.dtype == np.uint8 and cache.flags.c_contiguous and cache.shape[-1] == ROW_BYTES
    lat, lp = _c(latent, np.uint16)
    sl, sp = _c(slots, np.int64)
    assert lat.shape == (sl.shape[0], LATENT)
    rc = lib().oracle_store_fp8(lp, sp, sl.shape[0], cache.ctypes.data_as(C.c_void_p), cache.shape[0])
    if rc != 0:
        raise ValueError("slot past the end of the cache")


def dequant_rows_fp8(cache, rows) -> np.ndarray:
    cache = np.ascontiguousarray(cache, dtype=np.uint8).reshape(-1, ROW_BYTES)
    out = np.empty((len(rows), LATENT), dtype=np.float64)
    for i, r in enumerate(rows):
        lib().oracle_dequant_row_fp8(cache.ctypes.data_as(C.c_void_p), int(r), out[i].ctypes.data_as(C.c_void_p))
    return out


# ------------------------------------------------------------------------------------------------
# the 4-bit latent cache row (E2M1 codes, an E4M3 scale per 16 values, an fp32 scale per row;
# 304 bytes)
# ------------------------------------------------------------------------------------------------

FP4_ROW_BYTES = 304


def e2m1_value(code) -> float:
    return lib().oracle_e2m1_value(int(code) & 0xF)


def e2m1_encode(x) -> int:
    return int(lib().oracle_e2m1_encode(float(x)))


def store_fp4(latent, slots, cache) -> None:
    """Quantise ``latent`` (uint16 bf16 bits [n, 512]) into ``cache`` (uint8 [n_rows, 304]) in place."""
    assert cache.dtype == np.uint8 and cache.flags.c_contiguous and cache.shape[-1] == FP4_ROW_BYTES
    lat, lp = _c(latent, np.uint16)
    sl, sp = _c(slots, np.int64)
    assert lat.shape == (sl.shape[0], LATENT)
    rc = lib().oracle_store_fp4(lp, sp, sl.shape[0], cache.ctypes.data_as(C.c_void_p), cache.shape[0])
    if rc != 0:
        raise ValueError("slot past the end of the cache")


def dequant_rows_fp4(cache, rows) -> np.ndarray:
    cache = np.ascontiguousarray(cache, dtype=np.uint8).reshape(-1, FP4_ROW_BYTES)
    out = np.empty((len(rows), LATENT), dtype=np.float64)
    for i, r in enumerate(rows):
        lib().oracle_dequant_row_fp4(cache.ctypes.data_as(C.c_void_p), int(r), out[i].ctypes.data_as(C.c_void_p))
    return out


# ------------------------------------------------------------------------------------------------
# composition of the steps for one workload state (the order of the pages)
# ------------------------------------------------------------------------------------------------

def build_cache(inp, token_mask=None) -> np.ndarray:
    """store_int8 of every token (or of the tokens selected by ``token_mask``) into a fresh cache."""
    cache = np.zeros((inp.n_rows, ROW_BYTES), dtype=np.int8)
    if token_mask is None:
        store_int8(inp.latent, inp.slots, cache)
    else:
        store_int8(inp.latent[token_mask], inp.slots[token_mask], cache)
    return cache


def build_pools(inp) -> list:
    """pool_states of every sequence -> list of float64 [n_pools_b, 128]."""
    return [pool_states(inp.k[b], inp.gate[b], inp.pad[b], inp.len[b], inp.ln_w, inp.ln_b,
                        inp.wl.ln_eps) for b in range(inp.wl.batch)]


def decode_query(inp, n, cache, pools, select_k=None, out_width=None, pooled_override=None,
                 scores_override=None, attend=True) -> dict:
    """The whole hot path for query ``n``: index_scores -> topk_pools -> expand_selection ->
    rows through the slot map -> sparse MLA. ``pooled_override`` replaces the pooled keys of the
    query's sequence (e.g. the fp32 values a GPU consumed); ``scores_override`` replaces the
    scores fed to the selection."""
    wl = inp.wl
    S = wl.select_k if select_k is None else select_k
    W = wl.out_width if out_width is None else out_width
    b = int(inp.q_seq[n])
    pad, ln, qp = int(inp.pad[b]), int(inp.len[b]), int(inp.q_pos[n])
    pooled = pools[b] if pooled_override is None else pooled_override
    n_vis = n_visible_pools(pad, ln, qp)
    scores = index_scores(inp.q_idx[n], inp.w[n], pooled, n_vis)
    sel_scores = scores if scores_override is None else scores_override
    topk, n_sel = topk_pools(sel_scores, S)
    tok, n_valid = expand_selection(topk, n_sel, pad, ln, qp, W)
    rows = rows_from_tokens(tok, inp.slot_map[b])
    res = dict(n_vis=n_vis, scores=scores, topk=topk, n_sel=n_sel, tok=tok, n_valid=n_valid,
               rows=rows)
    if attend:
        res["out"], res["lse"] = sparse_mla(inp.q[n], cache, rows, inp.sm_scale)
    return res


# ------------------------------------------------------------------------------------------------
# context parallelism (TensorFold issue #402, 'Credit': local candidates merged into the global
# top-k; attention partials merged by log-sum-exp in rank order) -- definitions, in numpy fp64
# ------------------------------------------------------------------------------------------------

def merge_topk(cand_scores, cand_ids, select_k):
    """The select_k best of (score, id) candidates with distinct ids, by score descending and then
    the lower id (the order of topk_pools); -1 padded. Returns (ids int32 [select_k], count)."""
    s = np.asarray(cand_scores, dtype=np.float64).ravel()
    i = np.asarray(cand_ids, dtype=np.int64).ravel()
    keep = i >= 0
    s, i = s[keep], i[keep]
    s = np.where(s == 0.0, 0.0, s)                      # -0.0 ranks as +0.0
    order = np.lexsort((i, -s))                         # primary: score descending; then id
    n = min(int(select_k), len(order))
    out = np.full(int(select_k), INVALID, dtype=np.int32)
    out[:n] = i[order[:n]]
    return out, n


def lse_merge(outs, lses):
    """Attention over the union of disjoint row sets from each set's result: out_r [Hm, L] and
    lse_r [Hm] of parts r (taken in order; lse = -inf marks an empty part) ->
    LSE = log sum_r e^{lse_r}, out = sum_r e^{lse_r - LSE} out_r."""
    o = np.asarray(outs, dtype=np.float64)
    l = np.asarray(lses, dtype=np.float64)
    m = np.max(l, axis=0)
    safe = np.where(np.isfinite(m), m, 0.0)
    wgt = np.where(np.isfinite(l), np.exp(l - safe), 0.0)       # [parts, Hm]
    tot = wgt.sum(axis=0)
    out = np.einsum("rh,rhd->hd", wgt, o) / np.where(tot > 0, tot, 1.0)[:, None]
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return out, lse
