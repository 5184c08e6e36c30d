"""Micro-benchmark of the many-query entry points on one GPU (a prefill chunk's shapes).

    python kpool_indexer_int8_b200/microbench.py --op mla  --nq 1184 --reps 20
    python kpool_indexer_int8_b200/microbench.py --op gemm --nq 4096 --reps 10

--op mla:  glm_sparse_mla_decode on nq queries of 64 heads, each over 512 random pools of a
           135,168-row INT8 cache (2,048 rows as 4-row blocks, 3 tail rows, -1 padding to 2,176
           entries); random codes with row scales in [0.01, 0.05].
--op gemm: glm_index_scores_topk on nq causal queries at the end of a 135,168-token sequence
           (33,792 pools of N(0,1) fp32 keys), select_k 512.
Prints the CUDA-event time per call and the tensor-core rate it implies. With --reps 1 one call
runs after the warm-up, untimed (a single launch for a profiler).
"""
import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import kpool_indexer_int8_b200 as kp  # noqa: E402


def timed(fn, reps):
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    if reps <= 1:
        fn()
        torch.cuda.synchronize()
        return 0.0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1000.0 / reps


def mla(args, dev):
    torch.manual_seed(0)
    n_rows, W, nq, H = 135168, 2176, args.nq, 64
    cache = torch.randint(-127, 128, (n_rows, 528), dtype=torch.int8, device=dev)
    sc = (torch.rand(n_rows, device=dev) * 0.04 + 0.01).float()
    cache[:, 512:516] = sc.view(torch.int8).view(n_rows, 4)
    cache[:, 516:] = 0
    pools = torch.rand(nq, 33792, device=dev).topk(512, dim=1).indices.sort(dim=1).values
    rows = (pools[:, :, None] * 4 + torch.arange(4, device=dev)).reshape(nq, 2048)
    tail = torch.arange(n_rows - 3, n_rows, device=dev).expand(nq, 3)
    padr = torch.full((nq, W - 2051), -1, dtype=rows.dtype, device=dev)
    rows = torch.cat([rows, tail, padr], 1).to(torch.int32).contiguous()
    q = torch.randn(nq, H, 512, device=dev).to(torch.bfloat16)
    out = torch.empty(nq, H, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(nq, H, dtype=torch.float32, device=dev)
    dims = kp.make_dims(H)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_SPARSE_MLA, nq, width=W), dtype=torch.uint8, device=dev)
    fn = lambda: kp.glm_sparse_mla_decode(dims, q, cache, rows, 512 ** -0.5, out, ws, lse=lse)
    us = timed(fn, args.reps)
    flop = nq * H * 2051 * 512 * 2 * 2
    print(f"mla nq={nq}: {us:.1f} us per call, {flop / max(us, 1e-9) / 1e6:.1f} TFLOP/s (2 x q.k + p.v over 2051 rows)")


def gemm(args, dev):
    torch.manual_seed(0)
    nq, ld, S = args.nq, 33792, 512
    pooled = torch.randn(1, ld, 128, device=dev)
    qi = torch.randn(nq, 32, 128, device=dev).to(torch.bfloat16)
    w = torch.rand(nq, 32, device=dev)
    q_seq = torch.zeros(nq, dtype=torch.int32, device=dev)
    q_pos = torch.arange(4 * ld - nq, 4 * ld, dtype=torch.int32, device=dev)
    pad = torch.zeros(1, dtype=torch.int32, device=dev)
    length = torch.full((1,), 4 * ld, dtype=torch.int32, device=dev)
    topk = torch.empty(nq, S, dtype=torch.int32, device=dev)
    dims = kp.make_dims(64)
    ws = torch.empty(kp.glm_dsa_workspace_size(dims, kp.GLM_OP_INDEX_SCORES_TOPK, nq, ld, S), dtype=torch.uint8,
                     device=dev)
    fn = lambda: kp.glm_index_scores_topk(dims, qi, w, pooled, q_seq, q_pos, pad, length, S, topk, workspace=ws)
    us = timed(fn, args.reps)
    flop = nq * ld * 32 * 128 * 2 * 2
    print(f"index nq={nq}: {us:.1f} us per call (scores + selection), {flop / max(us, 1e-9) / 1e6:.1f} TFLOP/s of the two-term product")


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["mla", "gemm"], default="mla")
    ap.add_argument("--nq", type=int, default=1184)
    ap.add_argument("--reps", type=int, default=20)
    a = ap.parse_args()
    d = torch.device("cuda:0")
    {"mla": mla, "gemm": gemm}[a.op](a, d)
