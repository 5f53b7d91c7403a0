"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The hot path shards by independent work units (each GPU runs its own batch; no collective
on the data path), so the only cross-rank logic is the timing reduction (max over ranks),
the barrier around the timed region, the per-rank seeds and "rank 0 alone prints".
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    bench.init_dist(world, rank, backend="gloo")
    bench.barrier(world)
    # each rank reports its own times; everyone must see the element-wise maximum
    vals = bench.max_over_ranks([10.0 + rank, 5.0 - rank, float(rank)], world)
    seeds = (bench.rank_seed(rank, 0), bench.rank_seed(rank, 1))
    bench.barrier(world)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, vals, seeds))


def test_max_over_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, vals, _ in out:
        assert vals == [11.0, 5.0, 1.0]
    seeds = [s for _, _, s in out]
    assert len({s for pair in seeds for s in pair}) == 4  # distinct per rank and leg


def test_reference_arm_rank0_only_prints():
    # the oracle arm under two ranks: rank 0 prints one JSON line, rank 1 exits silently
    port = _free_port()
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2")
    outs = []
    for rank in (1, 0):
        e = dict(env, RANK=str(rank), LOCAL_RANK=str(rank))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--gpus", "2", "--steps", "1", "--warmup", "3"],
                           env=e, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    assert outs[0] == ""
    line = json.loads(outs[1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_window_pair_count():
    # the FLOP count of the sliding-window measurement: pairs (i, j) with i-W < j <= i
    sys.path.insert(0, ROOT)
    import bench
    for S, W in [(1, 1), (10, 3), (10, 10), (10, 0), (7, 20), (300, 64)]:
        brute = sum(1 for i in range(S) for j in range(S) if j <= i and (W == 0 or j > i - W))
        assert bench.window_pairs(S, W) == brute
