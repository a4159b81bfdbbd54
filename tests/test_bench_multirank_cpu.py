"""The bench's multi-rank host logic on CPU: two gloo ranks take distinct
shards, the timing reduction is a max over ranks, and the whole-job value
counts every rank's units over the slowest rank's time."""
import contextlib
import io
import json
import os
import socket
import time

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


RANK_SCRIPT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_bench_rank_cpu.py")


def test_spawn_ranks_runs_the_sharded_path_on_two_gloo_ranks(capfd):
    """bench.py --gpus 2 without torchrun: spawn_ranks starts one process per
    rank (the environment torchrun would give), each prepares and shards its
    workload as main() does, the step time is the max over ranks, and rank 0
    prints a line whose n_gpus is 2 and whose value counts both ranks' work."""
    argv = ["--gpus", "2", "--workload", "1", "--steps", "2", "--warmup", "3"]
    assert bench.spawn_ranks(2, argv, script=RANK_SCRIPT, timeout_s=300) == 0
    lines = [ln for ln in capfd.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                       # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2
    assert line["ms_per_step"] >= 20.0           # the slower rank's time
    assert abs(line["value"] - 2 * line["flops_per_rank"] / (line["ms_per_step"] * 1e-3) / 1e12) < 1e-12
    assert line["config"]["parallelism"] == "dp2 (independent shards)"
    c0, c1 = line["checksums"]
    assert c0 != c1                              # distinct shards
    w = build(1)                                 # rank 0 keeps the workload's own inputs
    assert abs(float(w.q.double().sum()) - c0[0]) < 1e-9
    # the reference arm reports the same config for the same workload
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(bench.parse_args(argv + ["--impl", "reference"]), rank=0)
    assert json.loads(buf.getvalue().strip().splitlines()[-1])["config"] == line["config"]


def test_spawn_ranks_stops_the_others_when_a_rank_fails(monkeypatch):
    monkeypatch.setenv("FAIL_RANK", "1")
    argv = ["--gpus", "2", "--workload", "1"]
    t0 = time.monotonic()
    assert bench.spawn_ranks(2, argv, script=RANK_SCRIPT, timeout_s=300) == 3
    assert time.monotonic() - t0 < 120           # rank 0 did not wait for its peer's timeout
