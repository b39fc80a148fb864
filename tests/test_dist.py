"""World-size-2 gloo checks of bench.py's multi-rank host logic (CPU only):
independent layer blocks are dealt to ranks without overlap, and every rank
reports the slowest rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = bench.blocks_for_rank(rank, world, 32)
        ms = bench.max_over_ranks(10.0 * (rank + 1), world)
        q.put((rank, mine, ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    blocks = res[0][1] + res[1][1]
    assert sorted(blocks) == list(range(32))
    assert not set(res[0][1]) & set(res[1][1])
    assert res[0][2] == res[1][2] == 20.0


def test_single_rank_helpers():
    assert bench.blocks_for_rank(0, 1, 3) == [0, 1, 2]
    assert bench.max_over_ranks(3.5, 1) == 3.5
