"""One rank of the 2-process CPU check of bench.py's cross-rank helpers (run under torchrun by
tests/test_multirank.py; not a test module itself)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bench  # noqa: E402


def main():
    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ["RANK"])
    bench.init_ranks(world, int(os.environ.get("LOCAL_RANK", "0")), need_gpu=False)
    try:
        # every rank takes the same collective steps in the same order
        torch.distributed.barrier()
        step_max = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
        e2e_max = bench.max_over_ranks(-float(rank), world, torch.device("cpu"))
        # one file per rank (the ranks' stdout streams interleave under the launcher)
        with open(os.path.join(sys.argv[1], f"rank{rank}.json"), "w") as f:
            json.dump({"rank": rank, "backend": torch.distributed.get_backend(), "step_max": step_max,
                       "e2e_max": e2e_max, "seed": bench.token_seed(rank)}, f)
    finally:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
