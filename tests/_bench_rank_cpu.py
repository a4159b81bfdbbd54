"""One rank of bench.py's multi-rank path on the CPU, as bench.spawn_ranks
starts it (RANK / WORLD_SIZE / MASTER_* in the environment, gloo): the same
argument parsing, per-rank workload preparation and sharding, max-over-ranks
reduction, whole-job value and config as bench.main(), with the kernel call
replaced by a host stand-in (a checksum of this rank's shard).  Rank 0 prints
one JSON line.  FAIL_RANK=r makes rank r exit with status 3 before joining."""
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bench  # noqa: E402


def main(argv):
    args = bench.parse_args(argv)
    rank, world, _ = bench.rank_env()
    if os.environ.get("FAIL_RANK") == str(rank):
        sys.exit(3)
    dist = bench.init_dist(world, "gloo")
    w = bench.prepare_workload(args, rank)
    flops_tiles, _ = bench.workload_flops(w, args.rope)
    t0 = time.perf_counter()
    checksum = torch.tensor([float(w.q.double().sum()), float(w.k.double().sum())], dtype=torch.float64)
    ms = (time.perf_counter() - t0) * 1e3 + 10.0 * (rank + 1)   # rank r: 10 (r + 1) ms and a bit
    (ms_max,) = bench.max_over_ranks([ms], dist, "cpu")
    sums = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
    if dist is not None:
        dist.all_gather(sums, checksum)
        dist.destroy_process_group()
    else:
        sums = [checksum]
    if rank == 0:
        print(json.dumps({"n_gpus": world, "ms_per_step": ms_max,
                          "value": bench.whole_job_tflops(flops_tiles, world, ms_max),
                          "flops_per_rank": flops_tiles, "config": bench.workload_config(w, world, args),
                          "checksums": [s.tolist() for s in sums]}), flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
