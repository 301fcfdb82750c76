"""The N > 1 host path of bench.py on CPU: two gloo ranks (the GPU run uses one rank per GPU over NCCL).

Checks what the ranks agree on without a GPU: each rank's expert shard (disjoint, covering the job), the timing
reduction (every rank gets the slowest rank's time) and the whole-job rate computed from it.
"""
import os
import socket
import sys
from datetime import timedelta

import multiprocessing as mp
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, experts, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    from synth import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        e0 = bench.rank_expert0(rank, experts)
        t = bench.max_over_ranks(torch, 10.0 + 3.0 * rank, world, torch.device("cpu"))
        rate = bench.whole_job_rate(world, 1.0e9, t)
        tags = [wl.tag(e0 + e, wl.W1) for e in range(experts)]
        q.put((rank, e0, t, rate, tags))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_shards_and_timing():
    world, experts = 2, 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, experts, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=240) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    # shards: rank r holds experts r*E .. r*E + E - 1; disjoint and together the whole job
    assert [r[1] for r in res] == [0, experts]
    all_tags = [t for r in res for t in r[4]]
    assert len(set(all_tags)) == world * experts
    import bench
    from synth import workloads as wl
    assert sorted(all_tags) == sorted(wl.tag(e, wl.W1) for e in range(world * experts))
    # timing: every rank reports the slowest rank's time, and the rate counts every rank's weights
    assert all(r[2] == 13.0 for r in res)
    assert all(abs(r[3] - world * 1.0e9 / 13.0 / 1e6) <= 1e-9 * r[3] for r in res)
    assert bench.whole_job_rate(1, 1.0e9, 13.0) * world == pytest.approx(res[0][3])
