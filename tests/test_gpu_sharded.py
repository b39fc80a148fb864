"""Row-sharded fit on one GPU: the shards run as threads, each on its own CUDA
stream with its own workspace, and a host-side reduction stands in for the
NCCL all-reduce (each shard's stream is synchronised before its buffer is
read, so no kernel ever waits on another shard's kernel).  Every reduced
quantity is an integer, so the sharded init, fit and pack must give the
unsharded call's results bit for bit: the same quantile tables, refined
tables, objective history and counters on every shard, and, concatenated
over the shards, the same codes, tagged scales and choice bits.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200 import synth

pytestmark = pytest.mark.gpu


class ThreadGroup:
    """All-reduce over shards running as host threads on one GPU."""

    def __init__(self, n):
        self.n = n
        self.bar = threading.Barrier(n, timeout=60)
        self.bufs = [None] * n

    def allreduce(self, rank):
        def run(t, op):
            torch.cuda.current_stream().synchronize()  # this shard's kernels are done
            self.bufs[rank] = t
            self.bar.wait()
            if rank == 0:
                acc = self.bufs[0].clone()
                for b in self.bufs[1:]:
                    acc = acc + b if op == "sum" else torch.maximum(acc, b)
                for b in self.bufs:
                    b.copy_(acc)
                torch.cuda.current_stream().synchronize()
            self.bar.wait()
        return run


def run_shards(W, I, cfg, splits):
    """init, fit and pack of W [N_total, K] split into row blocks of `splits`."""
    N_total = W.shape[0]
    group = ThreadGroup(len(splits))
    starts = np.cumsum([0] + list(splits))
    results = [None] * len(splits)
    errors = []

    def shard(rank):
        try:
            s = torch.cuda.Stream()
            c = bb.Config(cfg.fmt, cfg.g, cfg.S, cfg.iters, cfg.flags)
            with torch.cuda.stream(s):
                Ws = W[starts[rank]:starts[rank + 1]].contiguous()
                red = group.allreduce(rank)
                scales, T = bb.init_codebooks_sharded(Ws, N_total, c, red)
                T_init = T.clone()
                T, eh, st = bb.fit_layer_sharded(Ws, N_total, I, scales, T, c, red)
                out = bb.pack_sharded(Ws, N_total, I, scales, T, c, red)
                s.synchronize()
            results[rank] = dict(scales=scales, T_init=T_init, T=T, err_hist=eh, stats=st,
                                 gs=c.global_scale, **out)
        except Exception as e:  # surfaced below
            errors.append(e)
            group.bar.abort()

    threads = [threading.Thread(target=shard, args=(r,)) for r in range(len(splits))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    return results


CASES = [(bb.INT4, 128, 16, [37, 64, 27]), (bb.NVFP4, 16, 8, [50, 50]),
         (bb.NVFP4_GS, 16, 16, [1, 99, 28]), (bb.INT4, 128, 128, [128])]


@pytest.mark.parametrize("fmt,g,S,splits", CASES)
def test_sharded_equals_unsharded(fmt, g, S, splits):
    N, K, iters = sum(splits), 640, 5
    W, X = synth.small_layer(N, K, seed=N + S, T=64, heavy=True,
                             dist="normal" if fmt == bb.INT4 else "student_t4")
    W, X = W.cuda(), X.cuda()
    cfg = bb.Config(fmt, g, S, iters)
    ref = bb.run_layer(W, X, cfg)
    torch.cuda.synchronize()
    res = run_shards(W, ref["I"], cfg, splits)
    for r in res:
        assert torch.equal(r["T_init"], ref["T_init"])
        assert torch.equal(r["T"], ref["T"])
        assert torch.equal(r["err_hist"][:iters], ref["err_hist"][:iters])
        assert torch.equal(r["stats"], ref["stats"])
        assert torch.equal(r["T_bf16"], ref["T_bf16"])
        assert float(r["err_final"][0]) == float(ref["err_final"][0])
        if fmt == bb.NVFP4_GS:
            assert float(r["gs"][0]) == float(ref["global_scale"][0])
    for k in ("scales", "codes", "scales_tagged") + (("choice_bits",) if S != g else ()):
        assert torch.equal(torch.cat([r[k] for r in res]), ref[k]), k


def test_sharded_matches_the_oracle():
    """Three shards of an INT4 S=16 layer against the oracle's whole-layer run."""
    N, K, iters = 96, 512, 4
    W, X = synth.small_layer(N, K, seed=5, T=64, heavy=True)
    cfg = bb.Config(bb.INT4, 128, 16, iters)
    Wb = synth.bits_u16(W)
    ref = oracle.run_layer(Wb, synth.bits_u16(X), bb.INT4, 128, 16, iters)
    I = torch.from_numpy(ref["I"]).cuda()
    res = run_shards(W.cuda(), I, cfg, [40, 40, 16])
    assert np.array_equal(res[0]["T"].cpu().numpy().view(np.uint32), ref["T"].view(np.uint32))
    codes = torch.cat([r["codes"] for r in res]).cpu().numpy()
    assert np.array_equal(codes, ref["codes"])
    np.testing.assert_allclose(float(res[1]["err_final"][0]), ref["err_final"], rtol=1e-5)


def test_reduce_failure_is_reported():
    W = synth.make_weight(32, 256, 7).cuda()
    cfg = bb.Config(bb.INT4, 128, 16, 2)

    def broken(t, op):
        raise RuntimeError("peer lost")

    with pytest.raises(bb.AaacError, match="reduce callback failed"):
        bb.init_codebooks_sharded(W, 64, cfg, broken)
    torch.cuda.synchronize()


def test_sharded_fit_through_torch_distributed_nccl():
    """The torch.distributed adapter on a one-process NCCL group: the reduce
    buffers are views of the workspace handed to dist.all_reduce."""
    import os
    import socket

    import torch.distributed as dist
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        N, K = 64, 512
        W, X = synth.small_layer(N, K, seed=9, T=64, heavy=True)
        W, X = W.cuda(), X.cuda()
        cfg = bb.Config(bb.INT4, 128, 16, 3)
        ref = bb.run_layer(W, X, cfg)
        red = bb.torch_allreduce()
        scales, T = bb.init_codebooks_sharded(W, N, cfg, red)
        T, eh, st = bb.fit_layer_sharded(W, N, ref["I"], scales, T, cfg, red)
        out = bb.pack_sharded(W, N, ref["I"], scales, T, cfg, red)
        torch.cuda.synchronize()
        assert torch.equal(T, ref["T"]) and torch.equal(out["codes"], ref["codes"])
        assert torch.equal(eh[:3], ref["err_hist"][:3])
    finally:
        dist.destroy_process_group()
