"""The benchmark's multi-process plumbing on CPU (gloo, world size 2).

The EP ranks of the path are virtual partitions of one GPU, so bench.py runs
one independent replica per GPU: the only cross-process steps are the barrier
and the max over ranks of the timed region.  Those, and the rule that only rank
0 prints, are checked here without a GPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    ws, r, lr = bench.dist_env()
    d = bench.init_dist(ws, "gloo")
    dev = torch.device("cpu")
    bench.barrier(d, dev)
    m = bench.max_over_ranks(d, 1.5 + rank, dev)

    class A:
        steps, warmup, dispatch, seed = 2, 1, "dedup", 0
    line = bench.run_reference(A) if rank != 0 else None
    q.put((rank, ws, m, line))
    dist.destroy_process_group()


def test_max_over_ranks_and_rank_zero_only():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ws, m, line in out:
        assert ws == world
        assert m == pytest.approx(2.5)     # every rank sees the slowest rank's time
        assert line is None                # only rank 0 runs and prints the reference arm


def test_reference_arm_single_process():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup, dispatch, seed = 2, 1, "dedup", 0
    line = bench.run_reference(A)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
