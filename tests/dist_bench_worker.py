"""One rank of the two-rank (gloo, CPU) check of the benchmark's multi-rank
host logic; launched by tests/test_bench_ranks.py under
torch.distributed.run.  Prints one JSON line per rank."""
import datetime
import json
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    inp = bench.rank_inputs(rank, 64)
    cs = torch.tensor([float(np.asarray(inp["q"], np.float64).sum())], dtype=torch.float64)
    gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(gathered, cs)
    local_ms = 10.0 + 5.0 * rank
    mx = bench.max_over_ranks(local_ms, world, dist)
    value = bench.aggregate_tflops(world, 2e12, 4, mx)
    line = json.dumps({"rank": rank, "world": world, "checksums": [float(x) for x in gathered],
                       "local_ms": local_ms, "max_ms": mx, "value": value})
    for r in range(world):              # one rank at a time: the ranks share one stdout pipe
        if r == rank:
            print(line, flush=True)
        dist.barrier()
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
