"""Helper process for tests/test_multirank_cpu.py: started once per rank by
bench.py's replica launcher, it joins a gloo process group with the
environment the launcher set and writes what it saw to <outdir>/rank<R>.json."""
import datetime
import json
import os
import sys

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main(outdir):
    rank, world, local = bench.dist_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        t = torch.tensor([float(rank)])
        dist.all_reduce(t)   # every rank reached the group
        seen = dict(rank=rank, world=world, local=local, group_world=dist.get_world_size(),
                    rank_sum=float(t.item()), master=os.environ.get("MASTER_ADDR"),
                    max_over_ranks=bench.max_over_ranks(10.0 + rank, world))
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(seen, f)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main(sys.argv[1])
