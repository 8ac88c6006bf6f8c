"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks (world size 2).

Every rank decodes its own batch (requests are independent, so there is no data-path collective);
the step time is the max over ranks and the job throughput counts every rank's batch."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    t = bench.max_over_ranks(world, 1.5 + rank)           # ms of this rank's step
    seed = bench.rank_seed("long128k", rank)
    from sparse_attention_decode_sd_b200 import workloads as wl
    w = wl.make_workload(1, 4, 1, 64, 3, seed=seed)        # each rank's own small batch
    digest = float(w.q.float().sum())
    dist.barrier()
    out.put((rank, t, seed, digest, bench.job_tokens_per_s(world, 4, t)))
    dist.destroy_process_group()


def test_two_ranks_max_time_distinct_data_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, s0, d0, v0), (r1, t1, s1, d1, v1) = res
    assert t0 == t1 == 2.5                     # both ranks see the slowest rank's time
    assert s0 != s1 and d0 != d1               # different seeded batches
    assert v0 == v1 == pytest.approx(2 * 4 / 2.5e-3)
