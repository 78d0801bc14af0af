"""One rank of the multi-process host tests (gloo on CPU). Launched by
test_multiprocess.py with RANK / WORLD_SIZE / MASTER_ADDR / MASTER_PORT set;
prints one JSON line with what this rank observed."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    rank, world, local = bench.dist_setup()
    import torch.distributed as dist
    out = {"rank": rank, "world": world, "local": local, "backend": dist.get_backend()}
    # max over ranks of a per-rank step time (the bench takes the slowest rank)
    out["max"] = bench.dist_max(1.5 + rank, world)
    bench.barrier(world)
    # replicas: the reference arm runs on rank 0 only; other ranks return at once
    if rank != 0:
        class A:
            steps, warmup = 1, 3
        out["reference_rc"] = bench.run_reference(A, rank, world)
    bench.barrier(world)
    dist.destroy_process_group()
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
