"""The host side of sequence-sharded decode, on CPU with gloo (world size 2):
shard ranges tile the positions without gap or overlap, exactly one rank owns
the streaming heads, and the partials' exchange returns every rank's (o, lse)
in rank order.  The merge itself is a CUDA kernel, checked against the oracle
in tests/test_shard_gpu.py."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from head_split_kv_decode_b200 import shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_shard_ranges_tile_the_sequence():
    for cap, world in [(1000, 1), (1000, 3), (7, 4), (131072, 8)]:
        rs = shard.shard_ranges(cap, world)
        assert len(rs) == world and rs[0][0] == 0
        for (lo, hi), (lo2, _) in zip(rs, rs[1:]):
            assert lo < hi == lo2  # contiguous, no overlap
        assert rs[-1][1] >= cap
        assert sum(shard.owns_streaming(r) for r in range(world)) == 1


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        o = torch.full((2, 3, 4), float(rank + 1))       # [batch, Hq, d]
        lse = torch.full((2, 3), -float(rank))           # [batch, Hq]
        o_all, lse_all = shard.gather_partials(o, lse)
        q.put((rank, o_all, lse_all))
    finally:
        dist.destroy_process_group()


def test_gather_partials_in_rank_order():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, o_all, lse_all in results:
        assert o_all.shape == (2, 2, 3, 4) and lse_all.shape == (2, 2, 3)
        for r in range(world):
            assert torch.all(o_all[r] == r + 1) and torch.all(lse_all[r] == -r)
