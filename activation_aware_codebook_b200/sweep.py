"""Layer-parallel sweep of a multi-layer workload, with resume.

"Technical summary: AAAC", section 2 (efficiency: the fit needs only forward
activations and treats every layer on its own) -- so the (layer, linear)
units of a model are independent.  They are spread over ranks (one process
per GPU, ``torchrun``) with no collective: each rank fits and packs its own
units with libaaac and writes them; the host-side files are the only output.

Output directory:
  units/L{layer:02d}_{linear}.npz  T_bf16, codes, scales_tagged, choice_bits
                                   (when S < g), T, err_hist, stats
  manifest_r{rank}.jsonl           one JSON line per attempt:
                                   {"unit", "status": "ok"|"failed", "file",
                                    "sha256", "seconds", ...}
A result is written under a temporary name, renamed into place, and only
then recorded with status "ok" (line flushed and fsync'ed).  A unit counts as
done when some manifest line marks it "ok" and the named file exists with
the recorded sha256; a restart (any world size) skips done units and retries
failed or missing ones.

Partition: longest-processing-time first on the weight count N*K (ties by
layer, then the workload's linear order), each unit to the least-loaded rank;
a rank then runs its units in (layer, linear) order so that linears sharing
activations reuse one importance vector.

Command line (one process per GPU):
  torchrun --nproc-per-node 8 -m activation_aware_codebook_b200.sweep \\
      --workload llama8b-sweep-int4 --out /path/to/dir
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import time
from concurrent.futures import ThreadPoolExecutor
from typing import Callable, Dict, Iterable, List, Optional

import numpy as np

from . import synth


@dataclasses.dataclass(frozen=True)
class Unit:
    layer: int
    index: int  # position of the linear in the workload
    linear: synth.Linear

    @property
    def uid(self) -> str:
        return f"L{self.layer:02d}_{self.linear.name}"

    @property
    def weights(self) -> int:
        return self.linear.N * self.linear.K


def units_of(wl: synth.Workload, layers: Optional[Iterable[int]] = None,
             linears: Optional[Iterable[str]] = None) -> List[Unit]:
    layers = list(range(wl.layers)) if layers is None else list(layers)
    keep = None if linears is None else set(linears)
    return [Unit(l, i, lin) for l in layers for i, lin in enumerate(wl.linears)
            if keep is None or lin.name in keep]


def partition(units: List[Unit], world: int) -> List[List[Unit]]:
    """Longest-processing-time assignment by weight count; deterministic."""
    order = sorted(units, key=lambda u: (-u.weights, u.layer, u.index))
    load = [0] * world
    parts: List[List[Unit]] = [[] for _ in range(world)]
    for u in order:
        r = min(range(world), key=lambda i: (load[i], i))
        parts[r].append(u)
        load[r] += u.weights
    return [sorted(p, key=lambda u: (u.layer, u.index)) for p in parts]


def _sha256(path: str) -> str:
    h = hashlib.sha256()
    with open(path, "rb") as f:
        for chunk in iter(lambda: f.read(1 << 20), b""):
            h.update(chunk)
    return h.hexdigest()


def load_done(out_dir: str) -> Dict[str, dict]:
    """Units recorded "ok" whose file still matches its recorded hash."""
    done: Dict[str, dict] = {}
    if not os.path.isdir(out_dir):
        return done
    for name in sorted(os.listdir(out_dir)):
        if not (name.startswith("manifest_r") and name.endswith(".jsonl")):
            continue
        with open(os.path.join(out_dir, name)) as f:
            for line in f:
                try:
                    rec = json.loads(line)
                except json.JSONDecodeError:
                    continue  # a torn last line of an interrupted run
                if rec.get("status") != "ok":
                    continue
                path = os.path.join(out_dir, rec["file"])
                if os.path.exists(path) and _sha256(path) == rec.get("sha256"):
                    done[rec["unit"]] = rec
    return done


def _append(manifest: str, rec: dict) -> None:
    with open(manifest, "a") as f:
        f.write(json.dumps(rec) + "\n")
        f.flush()
        os.fsync(f.fileno())


def _save(out_dir: str, uid: str, arrays: Dict[str, np.ndarray]) -> str:
    rel = os.path.join("units", uid + ".npz")
    path = os.path.join(out_dir, rel)
    os.makedirs(os.path.dirname(path), exist_ok=True)
    tmp = path + f".tmp{os.getpid()}.npz"
    np.savez(tmp, **arrays)
    os.replace(tmp, path)
    return rel


Runner = Callable[[Unit], Dict[str, np.ndarray]]


def run_rank(out_dir: str, units: List[Unit], rank: int, world: int, runner: Runner,
             log: Optional[Callable[[str], None]] = None) -> dict:
    """Fit and store this rank's share of `units`, skipping done ones.  A
    unit's result is written by a background writer while the next unit
    runs on the GPU; the writer is the only thread that touches the files and
    the manifest, so the manifest keeps the units' order."""
    os.makedirs(out_dir, exist_ok=True)
    manifest = os.path.join(out_dir, f"manifest_r{rank}.jsonl")
    done = load_done(out_dir)
    mine = partition(units, world)[rank]
    skipped = 0
    t_all = time.time()
    writes = []

    def write_ok(u: Unit, arrays: Dict[str, np.ndarray], seconds: float) -> bool:
        try:
            rel = _save(out_dir, u.uid, arrays)
            _append(manifest, {"unit": u.uid, "status": "ok", "file": rel,
                               "sha256": _sha256(os.path.join(out_dir, rel)), "rank": rank,
                               "seconds": seconds, "N": u.linear.N, "K": u.linear.K})
            return True
        except Exception as e:  # recorded, retried by the next run
            write_failed(u, e)
            return False

    def write_failed(u: Unit, e: Exception) -> bool:
        _append(manifest, {"unit": u.uid, "status": "failed", "rank": rank,
                           "error": f"{type(e).__name__}: {e}"})
        if log:
            log(f"rank {rank}: {u.uid} failed: {e}")
        return False

    with ThreadPoolExecutor(max_workers=1) as writer:
        for u in mine:
            if u.uid in done:
                skipped += 1
                continue
            t0 = time.time()
            try:
                arrays = runner(u)
            except Exception as e:
                writes.append(writer.submit(write_failed, u, e))
                continue
            writes.append(writer.submit(write_ok, u, arrays, time.time() - t0))
        ok = [f.result() for f in writes]
    ran = sum(ok)
    return {"rank": rank, "world": world, "assigned": len(mine), "ran": ran,
            "skipped": skipped, "failed": len(ok) - ran, "seconds": time.time() - t_all,
            "weights": int(sum(u.weights for u in mine))}


def summary(out_dir: str, units: List[Unit]) -> dict:
    """Completion and the storage the learned tables add (section 2, core
    mechanism 3: about 64 bytes of BF16 table per layer)."""
    done = load_done(out_dir)
    table_bytes = 0
    for u in units:
        if u.uid in done:
            with np.load(os.path.join(out_dir, done[u.uid]["file"])) as z:
                table_bytes += z["T_bf16"].nbytes
    return {"units": len(units), "done": sum(u.uid in done for u in units),
            "table_bytes": int(table_bytes)}


def gpu_runner(wl: synth.Workload, tokens: int, iters: int, device) -> Runner:
    """importance -> init -> fit -> pack of one unit through libaaac; the
    importance vector of a (layer, activation key) is kept for the linears
    that share it."""
    import torch
    from . import binding as bb

    cfg = bb.Config(wl.fmt, wl.g, wl.S, iters)
    cache: Dict[tuple, torch.Tensor] = {}

    def run(u: Unit) -> Dict[str, np.ndarray]:
        lin = u.linear
        key = (u.layer, lin.x_key)
        if key not in cache:
            cache.clear()  # a rank walks layers in order: one layer's vectors at a time
        I = cache.get(key)
        if I is None:
            X = synth.make_activations(tokens, lin.K, synth.seed_of(wl.name, u.layer, lin.x_key, "X"),
                                       wl.heavy, device=device)
            I = bb.importance(X)
            del X
            cache[key] = I
        W = synth.make_weight(lin.N, lin.K, synth.seed_of(wl.name, u.layer, lin.name, "W"),
                              wl.w_dist, device=device)
        ws = bb.workspace(cfg, lin.N, lin.K, 0, device)
        scales, T = bb.init_codebooks(W, cfg, ws=ws)
        T, err_hist, stats = bb.fit_layer(W, I, scales, T, cfg, ws=ws)
        out = bb.pack(W, I, scales, T, cfg, ws=ws)
        torch.cuda.synchronize(device)
        arrays = {k: out[k].cpu().numpy() for k in ("T_bf16", "codes", "scales_tagged")}
        if out["choice_bits"] is not None:
            arrays["choice_bits"] = out["choice_bits"].cpu().numpy()
        arrays["T"] = T.cpu().numpy()
        arrays["err_hist"] = err_hist[:iters].cpu().numpy()
        arrays["err_final"] = out["err_final"].cpu().numpy()
        st = bb.decode_stats(stats)
        arrays["stats"] = np.array([st[k] for k in ("near_ties", "groups_t1", "empty_cells",
                                                    "dead_groups", "exact_groups", "L")],
                                   dtype=np.int64)
        return arrays

    return run


def main(argv=None) -> None:
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--workload", default="llama8b-sweep-int4")
    p.add_argument("--out", required=True)
    p.add_argument("--layers", type=int, default=0, help="first L layers only (0: all)")
    p.add_argument("--linears", default="", help="comma-separated subset of linear names")
    p.add_argument("--tokens", type=int, default=0, help="override calibration tokens")
    p.add_argument("--iters", type=int, default=0, help="override fit rounds")
    args = p.parse_args(argv)
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = synth.WORKLOADS[args.workload]
    units = units_of(wl, range(args.layers) if args.layers else None,
                     args.linears.split(",") if args.linears else None)
    runner = gpu_runner(wl, args.tokens or wl.tokens, args.iters or wl.iters, device)
    res = run_rank(args.out, units, rank, world, runner, log=print)
    res["workload"] = wl.name
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
