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


def _shard_reducer_rank(rank, world, port, out):
    import ctypes

    import torch
    import torch.distributed as dist

    from activation_aware_codebook_b200 import binding as bb
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ws = torch.zeros(256, dtype=torch.uint8)
    i64 = ws[64:64 + 4 * 8].view(torch.int64)
    i64.copy_(torch.tensor([rank + 1, -5 * rank, 7, 2 ** 40 * (rank + 1)]))
    i32 = ws[128:128 + 3 * 4].view(torch.int32)
    i32.copy_(torch.tensor([rank, 10 - rank, 3]))
    red = bb.ShardReducer(ws, bb.torch_allreduce())
    base = ws.data_ptr()
    rc = [red.fn(None, ctypes.c_void_p(base + 64), 4, bb.REDUCE_SUM_I64, None),
          red.fn(None, ctypes.c_void_p(base + 128), 3, bb.REDUCE_MAX_I32, None),
          red.fn(None, ctypes.c_void_p(base + 250), 4, bb.REDUCE_SUM_I64, None)]  # out of range
    torch.save({"rc": rc, "i64": i64.clone(), "i32": i32.clone()}, f"{out}/r{rank}.pt")
    dist.destroy_process_group()


def test_shard_reducer_over_gloo(tmp_path):
    """The adapter between the library's reduce callback and torch.distributed,
    run by two gloo ranks on CPU: sums and maxima land in place in the
    workspace views; a buffer outside the workspace is refused."""
    import torch
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_shard_reducer_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        d = torch.load(tmp_path / f"r{r}.pt")
        assert d["rc"] == [0, 0, 1]
        assert d["i64"].tolist() == [3, -5, 14, 3 * 2 ** 40]
        assert d["i32"].tolist() == [1, 10, 3]
