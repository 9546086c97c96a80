"""Multi-rank host logic on CPU: world-size-2 gloo process groups.

Covers the shard split (exact cover, alignment, balance), the deterministic
rank-ordered combine of parameter-gradient partials (identical bits on every
rank, equal to the fp64 rank-order sum), and the max-over-ranks timing
reduction.  No GPU: the exchange is the same torch.distributed call the NCCL
path makes.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from memory_efficient_activation_b200 import dist as mdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        g = np.random.Generator(np.random.Philox(key=[500 + rank, 0]))
        local = torch.from_numpy(g.normal(0.0, 1e3, size=288)).to(torch.float32)
        got = mdist.combine_param_grads(local)
        slow = mdist.max_over_ranks(float(rank) + 0.5)
        torch.save({"local": local, "got": got, "max": slow}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_combine_is_rank_ordered_and_identical(world, tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [torch.load(tmp_path / f"r{r}.pt") for r in range(world)]
    ref = res[0]["local"].double()
    for r in range(1, world):
        ref = ref + res[r]["local"].double()
    for r in range(world):
        assert torch.equal(res[r]["got"], ref.float())
        assert torch.equal(res[r]["got"], res[0]["got"])
        assert res[r]["max"] == world - 0.5


@pytest.mark.parametrize("n", [0, 1, 255, 256, 257, 67108864, 1000003])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_range_covers_exactly(n, world):
    prev_end = 0
    sizes = []
    for r in range(world):
        a, b = mdist.shard_range(n, r, world)
        assert a == prev_end
        assert a % mdist.SHARD_ALIGN == 0 or a == n
        prev_end = b
        sizes.append(b - a)
    assert prev_end == n
    assert max(sizes) - min(sizes) <= mdist.SHARD_ALIGN


def test_shard_range_rejects_bad_rank():
    with pytest.raises(ValueError):
        mdist.shard_range(10, 2, 2)
    with pytest.raises(ValueError):
        mdist.shard_range(-1, 0, 1)
