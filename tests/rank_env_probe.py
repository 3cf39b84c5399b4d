"""Stand-in for bench.py's per-rank work in the launcher test (no GPU): each
rank records the launcher's environment and its arguments, joins a gloo
process group and checks one all-reduce."""
import json
import os
import sys

import torch
import torch.distributed as dist


def main():
    out_dir = sys.argv[1]
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", init_method="env://")
    t = torch.tensor([float(rank + 1)])
    dist.all_reduce(t)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"rank": rank, "world": world, "local_rank": int(os.environ["LOCAL_RANK"]),
                   "master_addr": os.environ["MASTER_ADDR"], "sum": float(t.item()),
                   "argv": sys.argv[2:]}, f)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
