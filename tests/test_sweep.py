"""The layer-parallel sweep's host logic on CPU: partition, manifest, resume
after a failed unit, a corrupted result, a different world size, and the
storage the learned tables add ("Technical summary: AAAC", section 2, core
mechanism 3: about 64 bytes of BF16 tables per layer, about 14 KB for a 7B
model's 224 linears).  Two ranks run as gloo processes; the sweep itself has
no collective (layers are independent), the process group only provides the
barrier between the runs of a test.
"""
import json
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

from activation_aware_codebook_b200 import sweep, synth

WL = synth.WORKLOADS["llama8b-sweep-int4"]


def fake_runner(fail_marker=None, fail_uid=None, calls=None):
    def run(u):
        if calls is not None:
            with open(calls, "a") as f:
                f.write(u.uid + "\n")
        if fail_uid == u.uid and fail_marker and not os.path.exists(fail_marker):
            open(fail_marker, "w").close()
            raise RuntimeError("injected failure")
        seed = sum(map(ord, u.uid))
        return {"T_bf16": np.full((2, 16), seed, dtype=np.uint16),
                "codes": np.full((4, 8), seed & 255, dtype=np.uint8)}
    return run


def test_partition_covers_every_unit_once_and_balances():
    units = sweep.units_of(WL)
    assert len(units) == 32 * 7
    biggest = max(u.weights for u in units)
    for world in (1, 2, 3, 8):
        parts = sweep.partition(units, world)
        ids = [u.uid for p in parts for u in p]
        assert sorted(ids) == sorted(u.uid for u in units)
        loads = [sum(u.weights for u in p) for p in parts]
        assert max(loads) - min(loads) <= biggest
        assert parts == sweep.partition(units, world)  # deterministic
        for p in parts:  # layer order inside a rank
            assert [(u.layer, u.index) for u in p] == sorted((u.layer, u.index) for u in p)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir, marker, calls_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    units = sweep.units_of(WL, layers=range(2))
    calls = os.path.join(calls_dir, f"calls_{rank}.txt")
    res = sweep.run_rank(out_dir, units, rank, world,
                         fake_runner(marker, "L01_gate_proj", calls))
    with open(os.path.join(calls_dir, f"res_{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.barrier()
    dist.destroy_process_group()


def _run_world(world, out_dir, marker, calls_dir):
    mp.spawn(_rank_main, args=(world, _free_port(), out_dir, marker, calls_dir), nprocs=world,
             join=True)
    res = []
    for r in range(world):
        with open(os.path.join(calls_dir, f"res_{r}.json")) as f:
            res.append(json.load(f))
    return res


def test_resume_after_failure_two_ranks(tmp_path):
    out = str(tmp_path / "out")
    marker = str(tmp_path / "failed_once")
    units = sweep.units_of(WL, layers=range(2))
    calls_dir = str(tmp_path)
    # first run: every unit attempted once, one fails
    res = _run_world(2, out, marker, calls_dir)
    assert sum(r["ran"] for r in res) == len(units) - 1
    assert sum(r["failed"] for r in res) == 1
    done = sweep.load_done(out)
    assert set(done) == {u.uid for u in units} - {"L01_gate_proj"}
    # second run: only the failed unit runs
    for r in range(2):
        open(os.path.join(calls_dir, f"calls_{r}.txt"), "w").close()
    res = _run_world(2, out, marker, calls_dir)
    assert sum(r["ran"] for r in res) == 1 and sum(r["skipped"] for r in res) == len(units) - 1
    ran = [l.strip() for r in range(2)
           for l in open(os.path.join(calls_dir, f"calls_{r}.txt")) if l.strip()]
    assert ran == ["L01_gate_proj"]
    # a different world size resumes the same directory: nothing left to do
    res = sweep.run_rank(out, units, 0, 1, fake_runner())
    assert res["ran"] == 0 and res["skipped"] == len(units)
    # a corrupted result is detected by its hash and redone
    path = os.path.join(out, sweep.load_done(out)["L00_q_proj"]["file"])
    with open(path, "r+b") as f:
        f.seek(100)
        f.write(b"\xff\xff")
    assert "L00_q_proj" not in sweep.load_done(out)
    res = sweep.run_rank(out, units, 0, 1, fake_runner())
    assert res["ran"] == 1
    assert "L00_q_proj" in sweep.load_done(out)


def test_torn_manifest_line_is_ignored(tmp_path):
    out = str(tmp_path)
    units = sweep.units_of(WL, layers=range(1))
    sweep.run_rank(out, units, 0, 1, fake_runner())
    with open(os.path.join(out, "manifest_r0.jsonl"), "a") as f:
        f.write('{"unit": "L00_q_pr')  # an interrupted append
    assert len(sweep.load_done(out)) == len(units)


def test_table_storage_of_a_7b_sweep(tmp_path):
    """224 linears x two 16-entry BF16 tables = 224 x 64 B = 14,336 B, the
    page's "about 14 KB" for a 7B model."""
    units = sweep.units_of(WL)
    sweep.run_rank(str(tmp_path), units, 0, 1, fake_runner())
    s = sweep.summary(str(tmp_path), units)
    assert s["done"] == 224 and s["table_bytes"] == 224 * 64 == 14336
