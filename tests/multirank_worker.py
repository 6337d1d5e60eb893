"""Worker for test_multirank.py, launched by torch.distributed.run with the
gloo backend on CPU: every rank contributes rank + 1.5 to bench's
max-over-ranks reduction and checks the result."""
import os
import sys

import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def main():
    dist.init_process_group("gloo")
    rank, world = dist.get_rank(), dist.get_world_size()
    got = bench.max_over_ranks(rank + 1.5, world, "cpu")
    want = world - 1 + 1.5
    dist.barrier()
    print(f"rank {rank} max {got}", flush=True)
    dist.destroy_process_group()
    sys.exit(0 if got == want else 1)


if __name__ == "__main__":
    main()
