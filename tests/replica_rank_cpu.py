"""One rank of the CPU replica-launch test (run by bench.launch_replicas
under torch.distributed.run): joins a gloo group from the launcher's
environment, reports a rank-dependent device time through bench's
max-over-ranks and whole-job arithmetic, and rank 0 writes the result."""
import json
import os
import sys
from datetime import timedelta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main(out_path):
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(100.0 + 50.0 * rank, world, "cpu")
        value = bench.job_tokens_per_s(world, 3, 256, ms_max)
        if rank == 0:
            with open(out_path, "w") as f:
                json.dump({"world": world, "ms_max": ms_max, "value": value,
                           "local_rank": int(os.environ["LOCAL_RANK"])}, f)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main(sys.argv[1])
