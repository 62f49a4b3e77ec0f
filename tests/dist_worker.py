"""One rank of a torchrun-launched check of the bench's multi-rank plumbing
on the host (gloo): rendezvous from the environment, max over ranks, the
weak-scaling aggregate and per-rank seeds.  Each rank writes one JSON file,
rank<r>.json, into the directory given as the second argument."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    world, rank, local = bench.dist_setup(int(sys.argv[1]))
    try:
        bench.barrier(world)
        ms = 10.0 + 5.0 * rank          # rank r "took" 10 + 5r ms
        slowest = bench.max_over_ranks(ms, world)
        value = bench.whole_job_tflops(world, 2e12, slowest)
        bench.barrier(world)
        with open(os.path.join(sys.argv[2], "rank%d.json" % rank), "w") as f:
            json.dump({"rank": rank, "world": world, "local": local, "slowest_ms": slowest,
                       "value": value, "seed": bench.rank_seed(rank)}, f)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
