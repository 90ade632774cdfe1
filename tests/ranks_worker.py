"""One rank of the world-size-2 CPU test of bench.py's rank plumbing
(tests/test_bench_ranks.py launches two of these with torchrun on gloo).
Writes what this rank saw to <out_dir>/rank<r>.json."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402
from synthetic import workload_lengths  # noqa: E402

RAGGED = "ragged256_loguniform_1k_100k_d128_k64_bf16"


def main(out_dir: str) -> None:
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    local_rank = int(os.environ["LOCAL_RANK"])
    ranks = bench.init_rank_group(world, local_rank, "gloo")
    ranks.barrier()
    n = int(workload_lengths(RAGGED, bench.rank_seed(RAGGED, rank)).sum())
    seen = {
        "rank": rank,
        "world": world,
        "rows": n,
        "rows_total": ranks.sum(n),
        "max_time": ranks.max(10.0 + rank),
        "sum_ranks": ranks.sum(rank + 1),
    }
    ranks.barrier()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(seen, f)
    dist.destroy_process_group()


if __name__ == "__main__":
    main(sys.argv[1])
