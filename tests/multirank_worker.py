"""One rank of the two-rank CPU check of bench.py's multi-rank host path (gloo).

Run by tests/test_multirank_cpu.py through torch.distributed.run; each rank writes one
JSON file (rank<r>.json in the directory MULTIRANK_OUT) with the job time, the job
throughput and the rank's layer seed.
"""

import json
import os
import sys

import torch
import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def main() -> None:
    dist.init_process_group("gloo")
    try:
        rank, world = dist.get_rank(), dist.get_world_size()
        my_ms = 10.0 + 5.0 * rank                      # rank 1 is the slower one
        job_ms = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        value = bench.job_throughput(world, 4096 * 4096, 3, job_ms)
        dist.barrier()
        with open(os.path.join(os.environ["MULTIRANK_OUT"], f"rank{rank}.json"), "w") as f:
            json.dump({"rank": rank, "world": world, "job_ms": job_ms, "value": value,
                       "seed": bench.layer_seed(rank)}, f)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
