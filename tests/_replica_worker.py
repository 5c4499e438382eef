"""Worker for tests/test_replicas.py, launched by torch.distributed.run with the
gloo backend on CPU: exercises bench.py's replica aggregation (max over ranks,
whole-job rate) the way a multi-GPU bench run does, without a GPU."""
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def main():
    torch.distributed.init_process_group("gloo")
    rank, world = torch.distributed.get_rank(), torch.distributed.get_world_size()
    local_ms = 2.0 + 3.5 * rank  # the ranks finish at different times
    ms = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
    rate = bench.replica_rate(1000, ms, world)
    # one file per rank: the ranks share stdout, where their lines could interleave
    with open(os.path.join(os.environ["REPLICA_OUT"], f"rank{rank}.json"), "w") as f:
        json.dump({"rank": rank, "world": world, "local_ms": local_ms, "ms": ms, "rate": rate}, f)
    torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
