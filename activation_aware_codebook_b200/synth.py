"""Seeded synthetic layers and calibration activations.

This module only draws random inputs; it holds none of the fit's arithmetic,
and it serves both the CUDA path and the CPU oracle (the one thing the two
share).  The shapes and distributions stand in for the Llama / Qwen layers of
the AAAC evaluation ("Technical summary: AAAC", section 4: Llama 1B-13B and
Qwen 0.5B-32B, NVFP4 g=16 and INT4 g=128); no trained weights or datasets are
used.

Recipe (all draws fp32 from a seeded ``torch.Generator``, then bf16 RNE):
  W  ~ N(0, 0.02), or Student-t(nu=4) * 0.02 (t = z / sqrt(chi2_4 / 4), the
       chi-square made of four squared normals); then exactly
       round(0.001 * N * K) positions picked by a seeded randperm are
       multiplied by 10 ("0.1% outliers x10").
  X  = N(0, 1) * c_k with c_k = exp(N(0, 1)) per input column; "heavy" layers
       additionally multiply 5 seeded columns of c by 32.
  seed = crc32("<config>/<layer>/<linear>/<W|X>"), config 0 uses seed 0.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import List, Optional, Tuple

import torch

INT4 = 0
NVFP4 = 1
NVFP4_GS = 2  # NVFP4 with a per-tensor fp32 scale


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    N: int  # output rows
    K: int  # input columns (groups run along K)
    x_key: str  # linears that read the same activations share this key


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    linears: Tuple[Linear, ...]
    tokens: int
    w_dist: str  # "normal" | "student_t4"
    heavy: bool
    fmt: int
    g: int
    S: int
    iters: int
    layers: int = 1


def _llama8b(tokens: int) -> Tuple[Linear, ...]:
    return (
        Linear("q_proj", 4096, 4096, "attn_in"),
        Linear("k_proj", 1024, 4096, "attn_in"),
        Linear("v_proj", 1024, 4096, "attn_in"),
        Linear("o_proj", 4096, 4096, "attn_out"),
        Linear("gate_proj", 14336, 4096, "mlp_in"),
        Linear("up_proj", 14336, 4096, "mlp_in"),
        Linear("down_proj", 4096, 14336, "mlp_act"),
    )


WORKLOADS = {
    # single 256x512 layer, INT4 g=128 S=128, 10 iterations, seed 0
    "single-256x512-int4": Workload(
        "single-256x512-int4", (Linear("w", 256, 512, "x"),), 128, "normal", False, INT4,
        128, 128, 10),
    # Llama-3-1B-shaped linears (hidden 2048, MLP 8192), NVFP4 g=16, 20 iterations
    "llama1b-nvfp4": Workload(
        "llama1b-nvfp4",
        (Linear("attn_2048x2048", 2048, 2048, "h"), Linear("mlp_up_8192x2048", 8192, 2048, "h"),
         Linear("mlp_down_2048x8192", 2048, 8192, "a")),
        16384, "normal", True, NVFP4, 16, 16, 20),
    # Llama-3-8B-shaped q/k/v/o/gate/up/down, INT4 g=128 with S=16, 20 iterations
    "llama8b-int4-s16": Workload(
        "llama8b-int4-s16", _llama8b(262144), 262144, "normal", True, INT4, 128, 16, 20),
    # 32 layers x 7 linears of the 8B shapes, INT4 g=128 S=128, 20 iterations
    "llama8b-sweep-int4": Workload(
        "llama8b-sweep-int4", _llama8b(65536), 65536, "normal", True, INT4, 128, 128, 20,
        layers=32),
    # Qwen-32B-shaped largest projections, Student-t weights, NVFP4, 30 iterations
    "qwen32b-nvfp4": Workload(
        "qwen32b-nvfp4",
        (Linear("gate_27648x5120", 27648, 5120, "h"), Linear("up_27648x5120", 27648, 5120, "h"),
         Linear("down_5120x27648", 5120, 27648, "a")),
        131072, "student_t4", False, NVFP4, 16, 16, 30),
    # the same layers with NVFP4's per-tensor fp32 scale
    "qwen32b-nvfp4-gs": Workload(
        "qwen32b-nvfp4-gs",
        (Linear("gate_27648x5120", 27648, 5120, "h"), Linear("up_27648x5120", 27648, 5120, "h"),
         Linear("down_5120x27648", 5120, 27648, "a")),
        131072, "student_t4", False, NVFP4_GS, 16, 16, 30),
}


def seed_of(workload: str, layer: int, linear: str, what: str) -> int:
    if workload == "single-256x512-int4":
        return 0 if what == "W" else 1
    return zlib.crc32(f"{workload}/{layer}/{linear}/{what}".encode()) & 0x7FFFFFFF


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_weight(N: int, K: int, seed: int, dist: str = "normal", device="cpu",
                outlier_frac: float = 1e-3, outlier_mult: float = 10.0) -> torch.Tensor:
    """bf16 [N, K] weight drawn per the recipe in the module docstring."""
    g = _gen(seed, device)
    if dist == "normal":
        w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * 0.02
    elif dist == "student_t4":
        z = torch.randn(N, K, generator=g, device=device, dtype=torch.float32)
        chi = torch.zeros(N, K, device=device, dtype=torch.float32)
        for _ in range(4):
            e = torch.randn(N, K, generator=g, device=device, dtype=torch.float32)
            chi += e * e
        w = z / torch.sqrt(chi / 4.0) * 0.02
        del z, chi, e
    else:
        raise ValueError(dist)
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        idx = torch.randperm(N * K, generator=g, device=device)[:n_out]
        w.view(-1)[idx] *= outlier_mult
    return w.to(torch.bfloat16)


def channel_scales(K: int, seed: int, heavy: bool, device="cpu") -> torch.Tensor:
    g = _gen(seed ^ 0x5A5A5A5A, device)
    c = torch.exp(torch.randn(K, generator=g, device=device, dtype=torch.float32))
    if heavy:
        cols = torch.randperm(K, generator=g, device=device)[:5]
        c[cols] *= 32.0
    return c


def make_activations(T: int, K: int, seed: int, heavy: bool, device="cpu",
                     chunk_rows: int = 16384, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16 [T, K] calibration activations per the recipe (drawn in row chunks)."""
    c = channel_scales(K, seed, heavy, device)
    g = _gen(seed, device)
    X = out if out is not None else torch.empty(T, K, dtype=torch.bfloat16, device=device)
    for t0 in range(0, T, chunk_rows):
        t1 = min(T, t0 + chunk_rows)
        z = torch.randn(t1 - t0, K, generator=g, device=device, dtype=torch.float32)
        X[t0:t1] = (z * c).to(torch.bfloat16)
    return X


def bits_u16(t: torch.Tensor):
    """Raw bf16 bit patterns of a CPU tensor as a numpy uint16 array."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")


def small_layer(N: int, K: int, seed: int, T: int = 64, heavy: bool = False,
                dist: str = "normal", device="cpu"):
    """A small (W, X) pair for parity cases."""
    W = make_weight(N, K, seed, dist, device)
    X = make_activations(T, K, seed + 7919, heavy, device)
    return W, X


def linears_of(w: Workload) -> List[Linear]:
    return list(w.linears)
