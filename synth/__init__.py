"""Seeded synthetic inputs for the GLM-5.3-Flash kpool DSA decode path.

This module only draws random numbers and lays them out in memory. It holds none of the
method's arithmetic: no quantisation, no normalisation, no pool, tail or visibility rule.
Both sides take their inputs from here — the fp64 oracle (under ``oracle/``) and the CUDA
path (``kpool_indexer_int8_b200``) — and neither imports the other.

Random streams come from numpy's PCG64, one independent stream per tensor keyed by
``(seed, state, stream id)``, so a tensor's values do not depend on the sizes of the others.
BF16 tensors are returned as their raw 16-bit patterns (``uint16``); they are made by drawing
float32 samples and rounding them to the nearest bf16, ties to even.

Workload shapes follow the pages:
  * GLM-5.3 Kernels README ("Install the standalone kernels", "The tested MLA contract"):
    512-wide latents, 528-byte rows in blocks of 256, 16 query heads per rank, 2176 index slots,
    262,144-token contexts.
  * pypto-lib GLM-5.3-Flash page ("Checkpoint shape"): 64 attention heads, indexer 32 heads x 128,
    index_topk 2048, index_kpool 4, kv_lora_rank 512, qk_rope_head_dim 0.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

# Geometry fixed by the pages (pypto-lib "Checkpoint shape"; GLM-5.3 Kernels "Included").
KV_LORA_RANK = 512        # latent width L
INDEX_N_HEADS = 32        # indexer heads
INDEX_HEAD_DIM = 128      # indexer head dim
INDEX_KPOOL = 4           # tokens per pool
INDEX_TOPK = 2048         # selected tokens -> 512 pools
CACHE_BLOCK = 256         # rows per cache block
ROW_BYTES = 528           # 512 int8 + fp32 scale + 12 zero bytes

# stream ids (one independent random stream per tensor)
_S_LATENT, _S_OUTLIER, _S_K, _S_GATE, _S_LNW, _S_LNB, _S_QIDX, _S_W, _S_Q, _S_PERM, _S_JUNK, _S_LENS = range(12)


@dataclass(frozen=True)
class Workload:
    """A synthetic decode / prefill workload.

    Each sequence b has ``pads[b]`` left-padding positions followed by ``lens[b]`` valid tokens,
    in its own padded coordinates ``0 .. pads[b] + lens[b] - 1``. ``chunk == 0`` means one decode
    query per sequence at its last position; ``chunk > 0`` (batch 1 only) means ``chunk`` causal
    queries at the last ``chunk`` positions (a prefill chunk appended to the prefix).
    """
    name: str
    pads: tuple
    lens: tuple
    n_heads: int
    select_k: int
    out_width: int
    seed: int
    chunk: int = 0
    outlier_frac: float = 0.0
    outlier_scale: float = 8.0
    permute_slots: bool = False
    ln_eps: float = 1e-5

    @property
    def batch(self) -> int:
        return len(self.lens)

    @property
    def ld_tokens(self) -> int:
        return max(p + n for p, n in zip(self.pads, self.lens))

    @property
    def n_tokens(self) -> int:
        return int(sum(self.lens))

    @property
    def n_cache_rows(self) -> int:
        return -(-self.n_tokens // CACHE_BLOCK) * CACHE_BLOCK

    @property
    def n_queries(self) -> int:
        return self.chunk if self.chunk else self.batch


def _rng(seed: int, state: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, state, stream]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


# --------------------------------------------------------------------------------------------
# The five workloads (sizes from the pages; distributions as stated beside each)
# --------------------------------------------------------------------------------------------

TINY_DECODE = Workload("tiny_decode", pads=(0,), lens=(512,), n_heads=16, select_k=16,
                       out_width=80, seed=0)
PADDING_DECODE = Workload("padding_decode", pads=(0, 2, 3, 5), lens=(7, 64, 1027, 4096),
                          n_heads=64, select_k=512, out_width=2176, seed=1)
LONG_DECODE = Workload("long_decode", pads=(0,), lens=(262144,), n_heads=64, select_k=512,
                       out_width=2176, seed=2, outlier_frac=0.01)
CHUNKED_PREFILL = Workload("chunked_prefill", pads=(0,), lens=(131072 + 4096,), n_heads=64,
                           select_k=512, out_width=2176, seed=4, chunk=4096)


def batched_decode(seed: int = 3, batch: int = 8, lo: int = 32768, hi: int = 262144) -> Workload:
    """Batch of 8 with per-sequence contexts drawn uniformly from [lo, hi] and a randomly
    permuted slot mapping into one shared paged cache."""
    lens = _rng(seed, 0, _S_LENS).integers(lo, hi, size=batch, endpoint=True)
    return Workload("batched_decode", pads=(0,) * batch, lens=tuple(int(v) for v in lens),
                    n_heads=64, select_k=512, out_width=2176, seed=seed, permute_slots=True)


BATCHED_DECODE = batched_decode()

WORKLOADS = {w.name: w for w in (TINY_DECODE, PADDING_DECODE, LONG_DECODE, BATCHED_DECODE,
                                 CHUNKED_PREFILL)}


@dataclass
class Inputs:
    """Raw inputs of one workload state. BF16 tensors are uint16 bit patterns."""
    wl: Workload
    pad: np.ndarray          # int32 [B]      first valid position of each sequence
    len: np.ndarray          # int32 [B]      valid length of each sequence
    tok_start: np.ndarray    # int64 [B]      index in ``latent`` of each sequence's first valid token
    latent: np.ndarray       # uint16 [N_tok, 512]  bf16 MLA latents of the valid tokens, packed (b, t)
    slots: np.ndarray        # int64 [N_tok]   cache row of each packed token
    slot_map: np.ndarray     # int64 [B, ld]   cache row of token (b, t); -1 where there is none
    k: np.ndarray            # uint16 [B, ld, 128]  bf16 indexer keys (before k_norm)
    gate: np.ndarray         # uint16 [B, ld, 128]  bf16 pool gates
    ln_w: np.ndarray         # float32 [128]  k_norm weight
    ln_b: np.ndarray         # float32 [128]  k_norm bias
    q_seq: np.ndarray        # int32 [Nq]     sequence of each query
    q_pos: np.ndarray        # int32 [Nq]     padded position of each query
    q_idx: np.ndarray        # uint16 [Nq, 32, 128]  bf16 indexer queries
    w: np.ndarray            # float32 [Nq, 32]      indexer head weights
    q: np.ndarray            # uint16 [Nq, Hm, 512]  bf16 MLA queries (latent space)
    sm_scale: float = field(default=float(np.float32(KV_LORA_RANK ** -0.5)))

    @property
    def ld_tokens(self) -> int:
        return self.slot_map.shape[1]

    @property
    def n_rows(self) -> int:
        return self.wl.n_cache_rows

    def new_token_mask(self) -> np.ndarray:
        """bool [N_tok]: tokens the timed step writes (the query positions); the rest is the prefix."""
        m = np.zeros(self.latent.shape[0], dtype=bool)
        for qs, qp in zip(self.q_seq, self.q_pos):
            m[self.tok_start[qs] + (qp - self.pad[qs])] = True
        return m


def generate(wl: Workload, state: int = 0, junk_padding: bool = True) -> Inputs:
    """Draw all inputs of ``wl`` for independent state ``state`` (state 0 is the canonical one).

    Distributions: latents, q, q_idx, k, gate ~ N(0,1) (then bf16); a seeded ``outlier_frac`` of
    latent rows scaled by ``outlier_scale`` before rounding; w ~ U(0,1); k_norm weight ~ N(1, 0.1),
    bias ~ N(0, 0.1). Padding positions of k and gate hold junk of scale 1e4 unless
    ``junk_padding`` is False: no valid result may depend on them.
    """
    B, ld = wl.batch, wl.ld_tokens
    pad = np.asarray(wl.pads, dtype=np.int32)
    ln = np.asarray(wl.lens, dtype=np.int32)
    n_tok = wl.n_tokens
    tok_start = np.zeros(B, dtype=np.int64)
    tok_start[1:] = np.cumsum(ln.astype(np.int64))[:-1]
    s = wl.seed

    x = _rng(s, state, _S_LATENT).standard_normal(size=(n_tok, KV_LORA_RANK), dtype=np.float32)
    if wl.outlier_frac > 0:
        n_out = int(round(wl.outlier_frac * n_tok))
        rows = _rng(s, state, _S_OUTLIER).choice(n_tok, size=n_out, replace=False)
        x[rows] *= np.float32(wl.outlier_scale)
    latent = f32_to_bf16_bits(x)
    del x

    if wl.permute_slots:
        slots = _rng(s, state, _S_PERM).permutation(n_tok).astype(np.int64)
    else:
        slots = np.arange(n_tok, dtype=np.int64)
    slot_map = np.full((B, ld), -1, dtype=np.int64)
    for b in range(B):
        slot_map[b, pad[b]:pad[b] + ln[b]] = slots[tok_start[b]:tok_start[b] + ln[b]]

    k = _normal_bf16(_rng(s, state, _S_K), (B, ld, INDEX_HEAD_DIM))
    gate = _normal_bf16(_rng(s, state, _S_GATE), (B, ld, INDEX_HEAD_DIM))
    if junk_padding:
        jr = _rng(s, state, _S_JUNK)
        for b in range(B):
            for arr in (k, gate):
                if pad[b] > 0:
                    arr[b, :pad[b]] = _normal_bf16(jr, (pad[b], INDEX_HEAD_DIM), 1e4)
                end = pad[b] + ln[b]
                if end < ld:
                    arr[b, end:] = _normal_bf16(jr, (ld - end, INDEX_HEAD_DIM), 1e4)
    ln_w = (1.0 + 0.1 * _rng(s, state, _S_LNW).standard_normal(INDEX_HEAD_DIM)).astype(np.float32)
    ln_b = (0.1 * _rng(s, state, _S_LNB).standard_normal(INDEX_HEAD_DIM)).astype(np.float32)

    if wl.chunk:
        if B != 1:
            raise ValueError("a prefill chunk is defined for batch 1")
        end = int(pad[0] + ln[0])
        q_pos = np.arange(end - wl.chunk, end, dtype=np.int32)
        q_seq = np.zeros(wl.chunk, dtype=np.int32)
    else:
        q_pos = (pad + ln - 1).astype(np.int32)
        q_seq = np.arange(B, dtype=np.int32)
    nq = len(q_pos)
    q_idx = _normal_bf16(_rng(s, state, _S_QIDX), (nq, INDEX_N_HEADS, INDEX_HEAD_DIM))
    w = _rng(s, state, _S_W).random(size=(nq, INDEX_N_HEADS), dtype=np.float32)
    q = _normal_bf16(_rng(s, state, _S_Q), (nq, wl.n_heads, KV_LORA_RANK))

    return Inputs(wl=wl, pad=pad, len=ln, tok_start=tok_start, latent=latent, slots=slots,
                  slot_map=slot_map, k=k, gate=gate, ln_w=ln_w, ln_b=ln_b, q_seq=q_seq,
                  q_pos=q_pos, q_idx=q_idx, w=w, q=q)


def custom(name: str, pads, lens, n_heads: int = 16, select_k: int = 16, out_width: Optional[int] = None,
           seed: int = 100, **kw) -> Workload:
    """A small workload for parity tests (out_width defaults to 4*select_k + 3)."""
    if out_width is None:
        out_width = INDEX_KPOOL * select_k + INDEX_KPOOL - 1
    return Workload(name, pads=tuple(pads), lens=tuple(lens), n_heads=n_heads, select_k=select_k,
                    out_width=out_width, seed=seed, **kw)
