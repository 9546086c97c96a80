"""Stand-in worker for the launcher test of bench.py (tests/test_bench_launcher.py).

Run by bench._relaunch in place of bench.py: forms the process group from the
environment torch.distributed.run sets (gloo, CPU), takes the max over ranks
the way bench.py times its ranks, and rank 0 prints one JSON line with the
world size, the ranks the group formed and the arguments it was given.
"""
import datetime
import json
import os
import sys

import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from memory_efficient_activation_b200 import dist as mdist  # noqa: E402


def main():
    ws = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ["RANK"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    slowest = mdist.max_over_ranks(float(rank + 1), device="cpu")
    if rank == 0:
        print(json.dumps({"n_gpus": ws, "ranks_formed": dist.get_world_size(), "max_over_ranks": slowest,
                          "argv": sys.argv[1:]}), flush=True)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
