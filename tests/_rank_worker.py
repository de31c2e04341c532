"""One rank of a world-size-2 gloo job (launched by torchrun from
tests/test_multirank.py): bench.py's rank aggregation on the CPU.  Rank r
reports a timed region of 10 + 5 r ms and 1000 (r + 1) bytes; rank 0 prints
what every rank got back, one JSON line."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main():
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ms, units = bench.aggregate_ranks(10.0 + 5.0 * rank, 1000.0 * (rank + 1), world, "cpu")
        got = torch.tensor([ms, units], dtype=torch.float64)
        every = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(every, got)
        if rank == 0:
            print(json.dumps({"world": world, "per_rank": [e.tolist() for e in every]}), flush=True)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
