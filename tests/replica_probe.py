"""A stand-in for bench.py's per-rank work, used by test_multirank_cpu.py to drive
bench.maybe_relaunch: started with --gpus N outside torchrun, it re-executes itself
under torchrun; each gloo rank then reports a different elapsed time and rank 0 prints
the job time (the max over ranks) as one JSON line."""
import argparse
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=None)
    args = ap.parse_args()
    bench.maybe_relaunch(args.gpus, os.path.abspath(__file__), sys.argv[1:])
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        dist.init_process_group("gloo")
    ms = 10.0 + 5.0 * rank
    job_ms = bench.max_over_ranks(ms, dist if world > 1 else None, "cpu")
    if rank == 0:
        print(json.dumps({"world": world, "job_ms": job_ms,
                          "tops": bench.weak_scaling_tops(8.8e12, 3, world, job_ms)}))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
