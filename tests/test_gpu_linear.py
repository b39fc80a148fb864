"""GPU parity of the inference path on the packed format (reading R15):
aaac_dequant bit-exact against the oracle's bf16 dequantisation, and
aaac_linear within the fp32 summation bound K * 2^-24 * sum_k |x w_hat| of the
oracle's fp64 linear.  Packed layers come from the oracle's own pack, so the
inputs are independent of the CUDA fit.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200 import synth

pytestmark = pytest.mark.gpu


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32_of_bf16(h):
    return (np.asarray(h, dtype=np.uint32) << 16).view(np.float32)


def packed_layer(N, K, fmt, g, S, seed, iters=3, dist="normal"):
    """A layer fitted and packed by the oracle; returns (host dict, device dict).
    dev["cfg"] is the layer's config (with its tensor scale on the device for
    NVFP4_GS)."""
    W, X = synth.small_layer(N, K, seed, T=64, heavy=True, dist=dist)
    host = oracle.run_layer(u16(W), u16(X), fmt, g, S, iters)
    dev = {}
    for key in ("codes", "scales_tagged", "choice_bits", "T_bf16"):
        a = host[key]
        dev[key] = None if a is None else torch.from_numpy(
            np.ascontiguousarray(a).view(np.int16 if a.dtype == np.uint16 else a.dtype)).cuda()
    gs = (torch.tensor([host["gs"]], dtype=torch.float32).cuda() if fmt == oracle.NVFP4_GS
          else None)
    dev["cfg"] = bb.Config(fmt, g, S, 0, global_scale=gs)
    return host, dev


def ref_dequant(host, N, K, fmt, g, S):
    return oracle.dequant_bf16(host["codes"], host["scales_tagged"], host["choice_bits"],
                               host["T_bf16"], N, K, fmt, g, S, host["gs"])


CASES = [(oracle.INT4, 128, 16), (oracle.INT4, 128, 128), (oracle.INT4, 64, 8),
         (oracle.NVFP4, 16, 16), (oracle.NVFP4, 16, 8), (oracle.NVFP4_GS, 16, 16),
         (oracle.NVFP4_GS, 16, 8)]


@pytest.mark.parametrize("fmt,g,S", CASES)
@pytest.mark.parametrize("N,K", [(96, 512), (33, 384)])
def test_dequant_bit_exact(fmt, g, S, N, K):
    host, dev = packed_layer(N, K, fmt, g, S, seed=N + K + S)
    W_hat = bb.dequant(dev, dev["cfg"], N, K)
    assert np.array_equal(u16(W_hat), ref_dequant(host, N, K, fmt, g, S))


def check_linear(Y, Xb, Wh):
    ref = oracle.linear(Xb, Wh)
    K = Xb.shape[1]
    mag = np.abs(f32_of_bf16(Xb).astype(np.float64)) @ np.abs(f32_of_bf16(Wh).astype(np.float64)).T
    bound = K * 2.0 ** -24 * mag + 1e-30
    err = np.abs(Y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("fmt,g,S", CASES)
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 13])
def test_linear_within_bound(fmt, g, S, M):
    N, K = 70, 640
    host, dev = packed_layer(N, K, fmt, g, S, seed=7 + M)
    X = synth.make_activations(M, K, seed=100 + M, heavy=True).cuda()
    Y = bb.linear(X, dev, dev["cfg"], N, K)
    check_linear(Y, u16(X), ref_dequant(host, N, K, fmt, g, S))


def test_linear_strided_x_and_one_hot():
    N, K = 40, 256
    host, dev = packed_layer(N, K, oracle.INT4, 128, 16, seed=3)
    cfg = bb.Config(oracle.INT4, 128, 16, 0)
    wide = torch.zeros(4, K + 24, dtype=torch.bfloat16)
    cols = [0, 9, 130, 255]
    for i, c in enumerate(cols):
        wide[i, c] = 1.0
    Y = bb.linear(wide.cuda()[:, :K], dev, cfg, N, K)  # ldx = K + 24
    Wh = f32_of_bf16(oracle.dequant_bf16(host["codes"], host["scales_tagged"],
                                         host["choice_bits"], host["T_bf16"], N, K,
                                         oracle.INT4, 128, 16))
    for i, c in enumerate(cols):
        assert np.array_equal(Y[i].cpu().numpy(), Wh[:, c])


def test_dequant_and_linear_full_size_gate():
    """A 14336 x 4096 layer fitted and packed on the GPU; dequantisation
    bit-exact against the oracle on the same packed bits, and the M = 1 linear
    within the bound on every output."""
    N, K = 14336, 4096
    W = synth.make_weight(N, K, 91, device="cuda")
    X = synth.make_activations(2048, K, 92, True, device="cuda")
    cfg = bb.Config(oracle.INT4, 128, 16, 2)
    out = bb.run_layer(W, X, cfg)
    W_hat = bb.dequant(out, cfg, N, K)
    host = {k: (None if out[k] is None else out[k].cpu().numpy())
            for k in ("codes", "scales_tagged", "choice_bits", "T_bf16")}
    ref = oracle.dequant_bf16(host["codes"], host["scales_tagged"].view(np.uint16),
                              host["choice_bits"], host["T_bf16"].view(np.uint16), N, K,
                              oracle.INT4, 128, 16)
    assert np.array_equal(u16(W_hat), ref)
    x = synth.make_activations(1, K, 93, True, device="cuda")
    Y = bb.linear(x, out, cfg, N, K)
    check_linear(Y, u16(x), ref)


GEMM_CASES = [(oracle.INT4, 128, 16, 200, 640), (oracle.INT4, 128, 128, 130, 384),
              (oracle.NVFP4, 16, 16, 70, 208), (oracle.INT4, 32, 8, 256, 96),
              (oracle.NVFP4, 16, 8, 130, 176), (oracle.NVFP4_GS, 16, 16, 150, 272)]


@pytest.mark.parametrize("fmt,g,S,N,K", GEMM_CASES)
@pytest.mark.parametrize("M", [5, 9, 32, 64, 100, 257, 600])
def test_linear_tensor_core_path(fmt, g, S, N, K, M):
    """Token counts above 4 take the tcgen05 kernel: partial weight-row tiles
    (N not a multiple of 128), partial token tiles, and a last K block that
    is only partly inside K (K = 208, 96)."""
    host, dev = packed_layer(N, K, fmt, g, S, seed=M + N)
    X = synth.make_activations(M, K, seed=200 + M, heavy=True).cuda()
    Y = bb.linear(X, dev, dev["cfg"], N, K)
    torch.cuda.synchronize()
    assert bb.device_timeouts() == 0
    check_linear(Y, u16(X), ref_dequant(host, N, K, fmt, g, S))


@pytest.mark.parametrize("fmt,g,S", CASES)
@pytest.mark.parametrize("N,K,Ms", [(300, 4096, (1, 24, 64)), (130, 1024, (16, 40))])
def test_linear_small_token_counts(fmt, g, S, N, K, Ms):
    """1 to 64 tokens on a layer with many K blocks (K = 4096: 64 blocks, so
    every stage ring wraps many times) and partial weight-row tiles: the GEMV
    (1 token) and the fused tcgen05 kernel (its K split in two onto a zeroed
    Y); two runs agree bit for bit."""
    host, dev = packed_layer(N, K, fmt, g, S, seed=N + K + S + 5, iters=2)
    ref_w = ref_dequant(host, N, K, fmt, g, S)
    for M in Ms:
        X = synth.make_activations(M, K, seed=400 + M, heavy=True).cuda()
        Y = bb.linear(X, dev, dev["cfg"], N, K)
        Y2 = bb.linear(X, dev, dev["cfg"], N, K)
        torch.cuda.synchronize()
        assert bb.device_timeouts() == 0
        assert torch.equal(Y.view(torch.int32), Y2.view(torch.int32))
        check_linear(Y, u16(X), ref_w)


def test_linear_tensor_core_many_tiles():
    """150 weight-row tiles (at least one per SM): the unsplit path, each CTA
    over all of K."""
    N, K, M = 128 * 150, 128, 100
    host, dev = packed_layer(N, K, oracle.INT4, 128, 16, seed=11, iters=1)
    cfg = bb.Config(oracle.INT4, 128, 16, 0)
    X = synth.make_activations(M, K, seed=12, heavy=True).cuda()
    Y = bb.linear(X, dev, cfg, N, K)
    torch.cuda.synchronize()
    assert bb.device_timeouts() == 0
    Wh = oracle.dequant_bf16(host["codes"], host["scales_tagged"], host["choice_bits"],
                             host["T_bf16"], N, K, oracle.INT4, 128, 16)
    check_linear(Y, u16(X), Wh)


@pytest.mark.parametrize("fmt,g,S,N,K", GEMM_CASES)
@pytest.mark.parametrize("M", [192, 700])
def test_linear_dequantised_path(fmt, g, S, N, K, M):
    """From 192 tokens, aaac_linear_ws dequantises W once into its workspace
    and runs the TMA-fed tcgen05 GEMM: partial weight-row and token tiles and
    a K tail inside the last 64-wide block (K = 208, 96) come from the tensor
    maps' zero fill.  Within the same bound as the fused kernels."""
    host, dev = packed_layer(N, K, fmt, g, S, seed=M + N + 1)
    cfg = dev["cfg"]
    need = bb.linear_workspace_size(cfg, M, N, K)
    assert need >= N * K * 2
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    X = synth.make_activations(M, K, seed=300 + M, heavy=True).cuda()
    Y = bb.linear(X, dev, cfg, N, K, ws=ws)
    torch.cuda.synchronize()
    assert bb.device_timeouts() == 0
    check_linear(Y, u16(X), ref_dequant(host, N, K, fmt, g, S))
    # the workspace holds the dequantised weights, bit-exact
    assert np.array_equal(u16(ws[:N * K * 2].view(torch.int16).view(N, K)),
                          ref_dequant(host, N, K, fmt, g, S))


def test_linear_workspace_size_threshold():
    cfg = bb.Config(bb.INT4, 128, 16, 0)
    assert bb.linear_workspace_size(cfg, 191, 256, 512) == 0
    assert bb.linear_workspace_size(cfg, 192, 256, 512) >= 256 * 512 * 2
