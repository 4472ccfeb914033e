"""The multi-rank path of bench.py, on CPU with gloo (world size 2): each rank
runs a replica on distinct sequences, timings combine as the max over ranks,
and the whole-job rate counts every rank's bytes.  The reference arm under
torchrun prints exactly one line, from rank 0."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 30.0 - rank]          # per-rank (step ms, e2e ms)
        got = bench.max_over_ranks(mine, world, "cpu")
        ids = bench.replica_batch_ids(rank, 4)
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        q.put((rank, got, gathered))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_disjoint_replicas():
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
    for rank, got, gathered in results:
        assert got == [11.0, 30.0]               # element-wise max over ranks
        flat = [b for ids in gathered for b in ids]
        assert len(flat) == len(set(flat)) == 8   # replicas decode distinct rows


def test_aggregate_rate_counts_every_rank():
    # 2 ranks x 1e9 bytes per step x 10 steps in 20 ms -> 1000 GB/s
    assert bench.aggregate_rate(1e9, 2, 10, 20.0) == pytest.approx(1000.0)
    assert bench.aggregate_rate(1e9, 1, 10, 20.0) == pytest.approx(500.0)


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "tiny_mha_f32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
