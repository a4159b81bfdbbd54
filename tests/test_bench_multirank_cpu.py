"""The bench's multi-rank host logic on CPU: two gloo ranks take distinct
shards, the timing reduction is a max over ranks, and the whole-job value
counts every rank's units over the slowest rank's time."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import build


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.shard_workload(build(2, seq_scale=64), rank)
        checksum = torch.tensor([float(w.q.float().sum()), float(w.k.float().sum())])
        sums = [torch.zeros(2) for _ in range(world)]
        dist.all_gather(sums, checksum)
        ms = bench.max_over_ranks([1.0 + rank, 5.0 - rank], dist, "cpu")
        out[rank] = (sums, ms, bench.whole_job_tflops(1e12, world, ms[0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    sums0, ms0, v0 = out[0]
    sums1, ms1, v1 = out[1]
    assert not torch.equal(sums0[0], sums0[1])        # the two shards hold different data
    assert ms0 == ms1 == [2.0, 5.0]                   # max over ranks, the same on every rank
    assert abs(v0 - 1e12 * 2 / 2e-3 / 1e12) < 1e-9    # all ranks' units over the slowest time
    # rank 0 keeps the workload's own inputs
    w = build(2, seq_scale=64)
    assert abs(float(w.q.float().sum()) - float(sums0[0][0])) < 1e-3
