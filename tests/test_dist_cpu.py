"""The benchmark's multi-rank plumbing on CPU with the gloo backend, world size 2: replica states
are disjoint across ranks, the timing is the max over ranks, and the whole-job throughput counts
the units of every rank (weak scaling, no data-path collective)."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    my_ms = 10.0 + 5.0 * rank                       # rank 1 is the slower replica
    mx = bench.reduce_max(my_ms, world, "cpu")
    res = {"rank": rank, "max_ms": mx, "states": bench.replica_state_ids(rank, 8),
           "value": bench.whole_job_throughput(1, 100, world, mx)}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_replica_plumbing(tmp_path):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    assert r[0]["max_ms"] == r[1]["max_ms"] == 15.0
    assert not set(r[0]["states"]) & set(r[1]["states"])
    # 2 ranks x 100 steps x 1 query in 15 ms
    assert r[0]["value"] == pytest.approx(200 / 0.015)
