"""Stand-in for bench.py's GPU arm in the CPU test of its rank launcher.

It goes through bench.py's own launcher pieces: ``ensure_ranks`` (start one
rank per requested GPU under torch.distributed.run when not already a rank),
``rank_env``, ``max_over_ranks`` and ``emit``.  Each rank joins a ``gloo``
group and times a fixed host-side step whose length depends on its rank, so
that the reported time must be the slower rank's.  No GPU is used; this file
measures nothing about the library.
"""
import argparse
import datetime
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args()
    rc = bench.ensure_ranks(args.gpus, sys.argv[1:], os.path.abspath(__file__))
    if rc is not None:
        return rc
    import torch.distributed as dist
    world, rank, _ = bench.rank_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))

    def step():
        time.sleep(0.02 * (1 + rank))

    for _ in range(args.warmup):
        step()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    ms = (time.perf_counter() - t0) * 1e3
    total_ms = bench.max_over_ranks(ms, world, "cpu")
    bench.emit({"metric": "stub", "n_gpus": world, "steps": args.steps, "ms_per_step": total_ms / args.steps,
                "rank_ms_per_step": ms / args.steps}, rank)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
