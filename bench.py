#!/usr/bin/env python
"""Benchmark of the GLM-5.3-Flash kpool DSA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kernels|reference]
                    [--workload long_decode] [--states R]

One step = one pass of the whole path over one batch of the workload: store_int8 of the step's
new token(s) -> kpool_build of the pool(s) they complete -> index scores + top-k -> expand ->
sparse NoPE MLA (split + combine), all through the C ABI, replayed as one CUDA graph per
workload state. Inputs are synthetic (``synth``), resident in HBM before timing; R independent
states (each with its own cache, pooled keys and queries) are rotated so that no step finds the
previous step's bytes in L2 (8 x ~300 MB >> 126 MB of L2).

Multi-GPU (torchrun): replicas only -- each rank runs its own independent states (no data-path
collective); value = queries of all ranks / max-over-ranks time (weak scaling).

``--impl reference`` times the fp64 CPU oracle (the reference arm of this build) on a bounded
sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

# Kernels of one glm_dsa_decode_step: store + pool build + zeroing of the selection words, scores +
# top-k + expansion, MLA split, MLA combine.


def step_kernels(kp, wl, ld_pools: int, int8_keys: bool):
    """Kernels the one-call step enqueues for this workload (the library's own plan) and the names
    of its four stages (the step prefixes stop_after = 1, 2, 3 and the whole step)."""
    k, paths = kp.glm_dsa_step_plan(kp.make_dims(wl.n_heads), wl.n_queries, ld_pools, wl.batch, wl.out_width,
                                    int8_keys)
    names = ("step_prep",
             "index_qprep + index_gemm + topk_hist + topk_collect + expand" if paths & kp.GLM_PLAN_INDEX_MANY
             else "index_select_tc",
             "mla_multi_tc" if paths & kp.GLM_PLAN_MLA_MANY else "mla_split_tc",
             "mla_combine" if paths & kp.GLM_PLAN_MLA_COMBINE else "(no combine: mla_multi_tc writes the output)")
    return k, paths, names


def algorithmic_bytes(inp, key_bytes: int = 512, row_bytes: int = 528) -> dict:
    """Bytes the method must move per step (no partials, no score spills): each sequence's visible
    pooled keys once, its queries sharing them (512 B each, 132 for the INT8 indexer state), and
    per query q_idx + w and the top-k entries; each sequence's gathered cache rows once, at most
    its tokens (528 B each, 304 for 4-bit rows), and per query q + out and the indices; per step the
    store of the new rows and the pools they complete. With one query per sequence (decode) every
    term is that query's. `gathered` counts (query, row) pairs, the attention's work."""
    wl = inp.wl
    keys, rows = {}, {}   # per sequence: most visible pools of its queries, rows its queries gather
    per_q_idx = 0
    per_q_mla = 0
    gathered = 0
    for n in range(len(inp.q_pos)):
        s = int(inp.q_seq[n])
        upto = max(0, int(inp.q_pos[n]) - int(inp.pad[s]) + 1)
        n_vis = min(int(inp.len[s]), upto) // 4
        n_sel = min(n_vis, wl.select_k)
        tail = min(upto, int(inp.len[s])) - 4 * n_vis
        keys[s] = max(keys.get(s, 0), n_vis)
        rows[s] = rows.get(s, 0) + 4 * n_sel + tail
        per_q_idx += 32 * 128 * 2 + 32 * 4 + wl.select_k * 4
        per_q_mla += 2 * wl.n_heads * 512 * 2 + wl.out_width * 4
        gathered += 4 * n_sel + tail
    index = per_q_idx + sum(keys.values()) * key_bytes
    mla = per_q_mla + sum(min(r, int(inp.len[s])) for s, r in rows.items()) * row_bytes
    n_new = int(inp.new_token_mask().sum())
    store = n_new * (1024 + row_bytes + 8)
    new_pools = sum(1 for qs, qp in zip(inp.q_seq, inp.q_pos) if (qp - inp.pad[qs] + 1) % 4 == 0)
    kpool = new_pools * (4 * (256 + 256) + 512)
    return dict(index=index, mla=mla, store=store, kpool=kpool, gathered=gathered,
                total=index + mla + store + kpool)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense fp16/bf16 tensor TFLOP/s (the same rate for both 16-bit kinds): the measured burst
    figure (the kernel is timed over well under a second), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured bf16_tflops (burst)"
    return 1590.0, "fallback bf16_tflops (burst)"


def kernel_source_sha(name: str) -> str:
    """Hash of a kernel source file and of every local header it includes (recursively), so that
    a recorded counter goes stale when anything compiled into the kernel changes."""
    csrc = os.path.join(ROOT, "kpool_indexer_int8_b200", "csrc")
    h = hashlib.sha256()
    seen, todo = set(), [name]
    while todo:
        f = todo.pop(0)
        if f in seen:
            continue
        seen.add(f)
        path = os.path.join(csrc, f)
        if not os.path.exists(path):
            path = os.path.join(ROOT, "include", f)
        text = open(path, "rb").read()
        h.update(f.encode() + b"\0" + text)
        todo += re.findall(r'#include "([^"]+)"', text.decode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary, if the kernel's
    source has not changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel_file}:{workload}")
    if not d or d.get("source_sha") != kernel_source_sha(kernel_file):
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ------------------------------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)

    def _handle(self, device_index):
        import torch
        pynvml = self.nv
        uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            u = pynvml.nvmlDeviceGetUUID(h)
            u = u.decode() if isinstance(u, bytes) else u
            if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                return h
        return pynvml.nvmlDeviceGetHandleByIndex(device_index)

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "no samples")}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# the CPU oracle leg (cpu_baseline and --impl reference)
# ------------------------------------------------------------------------------------------------

def oracle_decode_throughput(wl, budget_s: float = 12.0, max_queries: int = 64, warmup: int = 0):
    """Time the fp64 oracle on decode queries of state 0 of the workload: per query the store of
    its new row, the pool that row completes, scores over all visible pools, top-k, expand and the
    sparse MLA. The oracle's state (cache, pools) is built beforehand, untimed, and `warmup`
    queries run untimed before the timed ones."""
    import oracle
    inp = synth.generate(wl, state=0)
    cache = oracle.build_cache(inp)
    pools = oracle.build_pools(inp)
    new = np.nonzero(inp.new_token_mask())[0]
    for w in range(warmup):
        oracle.decode_query(inp, w % len(inp.q_pos), cache, pools)
    done, t0 = 0, time.perf_counter()
    elapsed = 0.0
    while done < max_queries and (elapsed < budget_s or done == 0):
        n = done % len(inp.q_pos)
        s = int(inp.q_seq[n])
        t_new = new[n] if len(new) == len(inp.q_pos) else new[0]
        oracle.store_int8(inp.latent[t_new:t_new + 1], inp.slots[t_new:t_new + 1], cache)
        qp, pad = int(inp.q_pos[n]), int(inp.pad[s])
        if (qp - pad + 1) % 4 == 0:
            p = (qp - pad + 1) // 4 - 1
            t = pad + 4 * p
            pools[s][p] = oracle.pool_states(inp.k[s][t:t + 4], inp.gate[s][t:t + 4], 0, 4,
                                             inp.ln_w, inp.ln_b, wl.ln_eps)[0]
        oracle.decode_query(inp, n, cache, pools)
        done += 1
        elapsed = time.perf_counter() - t0
    return done / elapsed, done, elapsed


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # one reference step = one whole decode query of the oracle; K steps, cut at ~4 minutes
    qps, done, el = oracle_decode_throughput(wl, budget_s=240.0, max_queries=max(1, args.steps), warmup=args.warmup)
    line = {
        "impl": "reference", "metric": METRIC, "value": qps, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": done, "warmup": args.warmup,
        "ms_per_step": 1e3 / qps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, args),
        "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": 1, "kind": "oracle",
                         "sample": f"{done} decode queries of {wl.name} state 0 in {el:.1f} s"},
        "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "decode queries/s and achieved HBM GB/s (% of B200 peak), indexer+sparse MLA"


# ------------------------------------------------------------------------------------------------
# multi-rank plumbing (replicas only: no data-path collective)
# ------------------------------------------------------------------------------------------------

def replica_state_ids(rank: int, n_states: int) -> list:
    """Workload state ids of one rank: disjoint across ranks, so replicas never share inputs."""
    return [rank * n_states + r for r in range(n_states)]


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks of a per-rank time (the slowest replica bounds the whole job)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Units processed by all ranks divided by the max-over-ranks time (weak scaling)."""
    return units_per_rank_step * steps * world / (max_ms / 1e3)


def config_of(wl, args):
    return {"workload": wl.name, "batch": wl.batch, "context": list(wl.lens) if wl.batch > 1 else wl.lens[0],
            "queries_per_step": wl.n_queries, "n_heads": wl.n_heads, "select_k": wl.select_k,
            "out_width": wl.out_width, "kpool": 4, "index_heads": 32, "index_dim": 128,
            "latent": 512, "states": args.states,
            "pooled_keys": "int8 codes + fp32 scale per pool" if args.pooled == "int8" else "fp32",
            "latent_cache": {"int8": "int8 rows", "fp8": "fp8 (e4m3) rows",
                             "fp4": "4-bit rows (e2m1, e4m3 scale per 16)"}[args.cache],
            "l2": f"rotates {args.states} independent states per rank (inputs >> 126 MB L2)",
            "launch": f"one cuda graph of {args.states} steps (one per state) per replay", "parallelism": f"replicas x{args.gpus}"}


# ------------------------------------------------------------------------------------------------
# the CUDA path
# ------------------------------------------------------------------------------------------------

def run_kernels(args, wl):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    import kpool_indexer_int8_b200 as kp
    from kpool_indexer_int8_b200 import pipeline as P
    from synth import device as sdev

    R = args.states
    inps, bufs = [], []
    for r, sid in enumerate(replica_state_ids(rank, R)):
        inp = synth.generate(wl, state=sid)
        b = sdev.allocate_for(inp, dev, q8=args.pooled == "int8", fp8=args.cache == "fp8",
                               fp4=args.cache == "fp4")
        sdev.load(inp, b)
        bufs.append(b)
        inps.append(inp if r == 0 else None)
        del inp
    ab = algorithmic_bytes(inps[0], key_bytes=132 if args.pooled == "int8" else 512,
                           row_bytes=304 if args.cache == "fp4" else 528)
    n_kernels, paths, stage_names = step_kernels(kp, wl, bufs[0].pooled.shape[1], args.pooled == "int8")
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    if args.profile:
        # plain launches for a profiler: the one-call step (step_prep, index_select_tc,
        # mla_split_tc, mla_combine) or the separate entry points (store_int8, kpool_build,
        # index_select_tc, mla_split_tc, mla_combine) over the rotating states, no graphs, no timing
        fn = P.run_step if args.profile == "step" else P.run_stages
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                fn(bufs[i % R])
        stream.synchronize()
        if rank == 0:
            print(json.dumps({"profile": args.profile, "steps": args.steps, "workload": wl.name}), flush=True)
        return

    # one CUDA graph per state
    # one CUDA graph holding one step of every state in turn (R steps per replay, like a decode
    # graph over R layers), plus a one-step graph per state for a remainder of steps % R
    graphs = []
    with torch.cuda.stream(stream):
        for b in bufs:
            P.run_step(b)                       # eager once (idempotent step)
        stream.synchronize()
        multi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(multi, stream=stream):
            for b in bufs:
                P.run_step(b)
        for b in bufs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                P.run_step(b)
            graphs.append(g)
    torch.cuda.synchronize()

    def run_steps(k):
        for _ in range(k // R):
            multi.replay()
        for i in range(k % R):
            graphs[i].replay()

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up
    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    stream.synchronize()

    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        run_steps(args.steps)
        e1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    sampler.stop()
    barrier()
    ms = reduce_max(e0.elapsed_time(e1), world, dev)
    ms_per_step = ms / args.steps
    value = whole_job_throughput(wl.n_queries, args.steps, world, ms)

    # per-kernel cost inside the step: the same graphs of R steps cut after the step's first k
    # kernels (glm_dsa_decode_step's stop_after = k), timed the same way; kernel k's cost is the
    # difference of consecutive prefixes, so the costs add up to the whole step
    def time_graph(fn, reps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for b in bufs:
                fn(b)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for b in bufs:
                    fn(b)
            for _ in range(max(3, args.warmup // R + 1)):
                g.replay()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(reps):
                g.replay()
            a1.record(stream)
        stream.synchronize()
        t = a0.elapsed_time(a1) / (reps * R)
        del g
        return t

    reps = max(2, args.steps // R)
    prefix_ms = [time_graph(lambda b, k=k: P.run_step(b, stop_after=k), reps) for k in (1, 2, 3)]
    prefix_ms.append(time_graph(P.run_step, reps))
    kernel_ms = [prefix_ms[0]] + [prefix_ms[i] - prefix_ms[i - 1] for i in range(1, 4)]

    # the dominant kernel on its own: the fused scores + top-k + expansion entry over the rotating
    # states, captured as one graph and replayed (events on the launching stream); each launch moves
    # its query's pooled keys once, so the mean launch time gives the achieved GB/s
    idx_launch_ms = time_graph(P.index_topk_expand, reps)

    # end to end through the public API with host buffers: per step, one host->device copy of the
    # step's packed inputs (new latent rows and slots, q_idx, w, q, positions, pool begins) from
    # pinned memory, the new tokens' k and gate rows (one copy each per sequence), the one-call
    # step, and the output copied back device->host, then a synchronisation. Each state's copies
    # and step are captured as one CUDA graph, replayed in turn (the states rotate as above).
    import dataclasses
    e2e_fields = ("new_latent", "new_slots", "q_idx", "w", "q", "q_pos", "q_seq", "pool_begin")
    e2e = []
    for r, b in enumerate(bufs):
        srcs = [getattr(b, f) for f in e2e_fields]
        offs, total = [], 0
        for t in srcs:
            offs.append(total)
            total += (t.numel() * t.element_size() + 15) // 16 * 16
        d_pack = torch.empty(total, dtype=torch.uint8, device=dev)
        h_pack = torch.empty(total, dtype=torch.uint8).pin_memory()
        views = {}
        for f, t, o in zip(e2e_fields, srcs, offs):
            nb = t.numel() * t.element_size()
            views[f] = d_pack[o:o + nb].view(t.dtype).view(t.shape)
            h_pack[o:o + nb].copy_(t.reshape(-1).view(torch.uint8).cpu())
        b2 = dataclasses.replace(b, **views)
        q_seq_h, q_pos_h = b.q_seq.cpu().numpy(), b.q_pos.cpu().numpy()
        kg = []
        for sq in sorted(set(int(v) for v in q_seq_h)):
            pos = q_pos_h[q_seq_h == sq]
            lo_t, hi_t = int(pos.min()), int(pos.max()) + 1
            kg.append((b.k[sq, lo_t:hi_t], b.k[sq, lo_t:hi_t].cpu().pin_memory(),
                       b.gate[sq, lo_t:hi_t], b.gate[sq, lo_t:hi_t].cpu().pin_memory()))
        h_out = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()
        e2e.append((b2, d_pack, h_pack, kg, h_out))
    h2d = e2e[0][1].numel() + sum(hk.numel() * hk.element_size() + hg.numel() * hg.element_size()
                                  for _, hk, _, hg in e2e[0][3])
    d2h = e2e[0][4].numel() * e2e[0][4].element_size()

    def e2e_step(item):
        b2, d_pack, h_pack, kg, h_out = item
        d_pack.copy_(h_pack, non_blocking=True)
        for dk, hk, dg, hg in kg:
            dk.copy_(hk, non_blocking=True)
            dg.copy_(hg, non_blocking=True)
        P.run_step(b2)
        h_out.copy_(b2.out, non_blocking=True)

    e2e_graphs = []
    with torch.cuda.stream(stream):
        for item in e2e:
            e2e_step(item)
        stream.synchronize()
        for item in e2e:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                e2e_step(item)
            e2e_graphs.append(g)
        for g in e2e_graphs:
            g.replay()
        stream.synchronize()
    n_e2e = max(R, min(args.steps, 400))
    done = torch.cuda.Event()                    # (no timing: query() polls it)
    with torch.cuda.stream(stream):              # replays go to the stream the graphs were captured on
        t0 = time.perf_counter()
        for i in range(n_e2e):
            e2e_graphs[i % R].replay()
            done.record(stream)
            while not done.query():              # the host waits for the output by polling, as a
                pass                             # latency-bound serving loop would
        e2e_s = time.perf_counter() - t0
    assert torch.equal(e2e[(n_e2e - 1) % R][4], e2e[(n_e2e - 1) % R][0].out.cpu())   # the copy is the output
    e2e_qps = whole_job_throughput(wl.n_queries, n_e2e, world, reduce_max(e2e_s * 1e3, world, dev))
    del e2e_graphs

    peak, peak_kind = measured_peaks()
    if paths & kp.GLM_PLAN_MLA_MANY and kernel_ms[2] >= max(kernel_ms):
        # dominant kernel: the walking attention (many queries), a tensor-core contraction:
        # q . k and p . v over every gathered row, 2 x 2 x 512 FLOP per (row, head)
        flop = ab["gathered"] * wl.n_heads * 512 * 2 * 2
        t_peak, t_kind = measured_tensor_peak()
        mla_s = kernel_ms[2] / 1e3
        roofline = {"kernel": "mla_multi_tc (walking attention; its share of the step, step prefixes)",
                    "bound": "tensor", "achieved": flop / mla_s / 1e12, "peak": t_peak, "peak_kind": t_kind,
                    "unit": "TFLOP/s", "frac": flop / mla_s / 1e12 / t_peak, "traffic": None,
                    "algorithmic_flop_per_launch": flop, "launch_us": kernel_ms[2] * 1e3}
    else:
        # dominant kernel: the fused scores + selection + expansion launch (each timed launch also
        # carries the tiny zeroing launch of the multi-CTA selection words)
        idx_ms = idx_launch_ms
        achieved = ab["index"] / (idx_ms / 1e3) / 1e9
        traffic = recorded_traffic("index_select_tc.cu", wl.name + ("_q8" if args.pooled == "int8" else ""))
        roofline = {"kernel": "index_select_tc (scores + top-k + expansion)", "bound": "hbm", "achieved": achieved,
                    "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s", "frac": achieved / peak,
                    "traffic": traffic, "algorithmic_bytes_per_launch": ab["index"],
                    "launch_us": idx_ms * 1e3}
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "precision": "int8 (or fp8) cache rows and bf16 tensor-core operands, fp32 accumulation",
        "data": "synthetic", "config": config_of(wl, args),
        "achieved_hbm_gbs_per_gpu": ab["total"] / (ms_per_step / 1e3) / 1e9,
        "algorithmic_bytes_per_step": ab["total"],
        "tokens_gathered_per_s": ab["gathered"] * args.steps * world / (ms / 1e3),
        "kernel_us_in_step": {nm: v * 1e3 for nm, v in zip(stage_names, kernel_ms)},
        "kernel_us_method": "step prefixes (stop_after = 1, 2, 3, whole) as graphs of the rotating states; "
                            "each kernel = difference of consecutive prefixes; their sum is the whole step "
                            f"timed the same way ({prefix_ms[3] * 1e3:.2f} us)",
        "roofline": roofline,
        "e2e": {"value": e2e_qps, "unit": "queries/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": n_e2e,
                "api": "glm_dsa_decode_step through the binding with its host copies (pinned, one packed "
                       "H2D of the step inputs + the new k/gate rows, one D2H of out) captured per state "
                       "as a CUDA graph, replayed per step; the host waits for each step's output by "
                       "polling an event recorded after it"},
        "gpu_launches": n_kernels * args.steps,
        "clocks": sampler.summary(),
    }
    line["achieved_hbm_frac_per_gpu"] = line["achieved_hbm_gbs_per_gpu"] / peak
    if world == 1 and rank == 0 and not args.no_cpu_baseline and args.cache == "int8":
        qps, done, el = oracle_decode_throughput(wl, budget_s=12.0)
        line["cpu_baseline"] = {"value": qps, "unit": "queries/s", "cores": 1, "kind": "oracle",
                                "sample": f"{done} decode queries of {wl.name} state 0 ({el:.1f} s); oracle state built untimed"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs, multi
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["kernels", "reference"], default="kernels")
    ap.add_argument("--workload", default="long_decode", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--states", type=int, default=8)
    ap.add_argument("--pooled", choices=["fp32", "int8"], default="fp32",
                    help="indexer state: fp32 pooled keys (the pages' path) or the INT8 variant")
    ap.add_argument("--cache", choices=["int8", "fp8", "fp4"], default="int8",
                    help="latent cache rows: INT8 (the pages' path) or the FP8 or 4-bit variant")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["step", "stages"], default=None,
                    help="run --steps plain launches (no graphs, no timing) for a profiler and exit")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_kernels(args, wl)


if __name__ == "__main__":
    sys.exit(main())
