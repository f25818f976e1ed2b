"""Worker for the multi-rank CPU tests (launched by torch.distributed.run with
the gloo backend): exercises bench.py's max-over-ranks timing reduction and
its whole-job rate the way the N-GPU bench uses them, with per-rank timings
that differ on purpose."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main():
    out_dir = sys.argv[1]
    rank, world, _ = bench.dist_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    # rank r "took" 100 + 25 r ms for 50 steps and 7 - r ms end to end
    mine = [100.0 + 25.0 * rank, 7.0 - rank]
    dist.barrier()
    ms, e2e = bench.max_over_ranks(mine, world, "cpu")
    rate = bench.job_rate(50, world, ms)
    dist.barrier()
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump({"rank": rank, "world": world, "mine": mine, "ms": ms, "e2e": e2e, "rate": rate}, f)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
