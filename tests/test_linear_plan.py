"""The W4A16 linear's choice of kernel and the cluster kernel's plan (host
code, no GPU), from aaac_linear_launch_plan.

aaac_linear takes the GEMV up to 4 tokens, the cluster kernel (2 to 8 CTAs
split a 128-row tile's 64-column K blocks, about 240 CTAs in all; the rows'
scales and choice bits of a CTA's K range are staged in shared memory) from 5
to 32 tokens when K is a
multiple of 32 and that staging fits, and the fused tcgen05 kernel otherwise.
The emulation below takes each CTA's share of the K blocks as the kernel does
(CTA r of C: blocks [r*nkb/C, (r+1)*nkb/C)) and checks that the shares cover
every block once, that every CTA has a block, and that the scale groups and
choice-bit bytes a CTA touches fit the staged rows.
"""
import pytest
import torch

from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200.csrc import build as cbuild


@pytest.fixture(scope="module", autouse=True)
def lib():
    cbuild.build()
    return bb.load()


CFGS = [(bb.INT4, 128, 16), (bb.INT4, 128, 128), (bb.INT4, 64, 8), (bb.INT4, 32, 8),
        (bb.NVFP4, 16, 16), (bb.NVFP4, 16, 8), (bb.NVFP4_GS, 16, 16)]
SHAPES = [(70, 640), (256, 96), (130, 384), (14336, 4096), (4096, 14336), (1024, 4096),
          (5120, 27648), (27648, 5120), (200, 208), (130, 176), (40, 256), (8, 65536)]


def _emulate(p, K, g, S):
    C, nkb = p["cluster"], p["kblocks"]
    esz = 1 if p["fmt"] != bb.INT4 else 2
    seen = []
    for r in range(C):
        lo, hi = r * nkb // C, (r + 1) * nkb // C
        assert hi > lo, "a CTA without K blocks"
        seen.extend(range(lo, hi))
        col_lo, col_hi = lo * 64, min(K, hi * 64)
        groups = (col_hi - 1) // g - col_lo // g + 1
        assert groups * esz <= p["scale_stride"]
        if S != g:
            nbytes = ((col_hi - 1) // S) // 8 - (col_lo // S) // 8 + 1
            assert nbytes <= p["choice_stride"]
        else:
            assert p["choice_stride"] == 0
    assert seen == list(range(nkb)), "K blocks not covered exactly once"


@pytest.mark.parametrize("fmt,g,S", CFGS)
@pytest.mark.parametrize("N,K", SHAPES)
def test_linear_path_and_cluster_plan(fmt, g, S, N, K):
    if K % g:
        pytest.skip("K not a multiple of g")
    # the plan never reads the tensor scale; a host tensor stands for it
    gs = torch.zeros(1, dtype=torch.float32) if fmt == bb.NVFP4_GS else None
    cfg = bb.Config(fmt, g, S, 0, global_scale=gs)
    for M in (1, 4, 5, 16, 17, 32, 33, 64, 191):
        p = bb.linear_launch_plan(cfg, M, N, K)
        p["fmt"] = fmt
        assert p["kblocks"] == (K + 63) // 64
        tiles = (N + 127) // 128  # about 240 CTAs, 2 to 8 a cluster, at most the K blocks
        assert p["cluster"] == min(max(2, min(8, (240 + tiles // 2) // tiles)), p["kblocks"])
        fits = p["smem32"] <= p["smem_limit"]
        assert p["smem16"] <= p["smem32"]
        if M <= 4:
            assert p["path"] == "gemv"
        elif M <= 32 and K % 32 == 0 and fits:
            assert p["path"] == "cluster"
        else:
            assert p["path"] == "fused"
        _emulate(p, K, g, S)


def test_wide_nvfp4_layer_falls_back_to_the_fused_kernel():
    """NVFP4 g=16 with K = 27648 and S = 8 on a layer of 216 row tiles (two
    CTAs a cluster): a CTA's half of K stages 866 scale bytes and 110 choice
    bytes per row, past shared memory at 32 tokens."""
    p = bb.linear_launch_plan(bb.Config(bb.NVFP4, 16, 8, 0), 16, 27648, 27648)
    assert p["cluster"] == 2
    assert p["smem32"] > p["smem_limit"]
    assert p["path"] == "fused"


def test_linear_plan_rejects_bad_arguments():
    cfg = bb.Config(bb.INT4, 128, 16, 0)
    with pytest.raises(RuntimeError):
        bb.linear_launch_plan(cfg, 0, 128, 512)
    with pytest.raises(RuntimeError):
        bb.linear_launch_plan(cfg, 4, 128, 500)  # K not a multiple of g
