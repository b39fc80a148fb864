"""GPU parity of the AWQ-style pre-scaling and of the device-side grid search
("Technical summary: AAAC", section 4: AAAC combined with AWQ's scaling of the
weights before quantisation; reading R16 for the scaling).  c, I' and W' are
bit-exact against the oracle; the search's packed output, kept position and
scales are bit-exact against the oracle's search, and each candidate's
err_final is within the objective tolerance.  Inputs come from the seeded
generators; importance vectors are computed by the oracle (or drawn directly),
never by the CUDA path.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200 import synth

pytestmark = pytest.mark.gpu

RTOL = 1e-5


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32bits(t):
    return t.detach().cpu().numpy().view(np.uint32)


def _layer(N, K, seed, T=64, dist="normal"):
    W, X = synth.small_layer(N, K, seed, T=T, heavy=True, dist=dist)
    return W, synth.bits_u16(W), synth.bits_u16(X)


@pytest.mark.parametrize("N,K", [(33, 1040), (64, 512), (5, 24)])
@pytest.mark.parametrize("j", [0, 1, 7, 8, 13, 16])
def test_prescale_bit_exact(N, K, j):
    W, Wb, Xb = _layer(N, K, seed=N + K + j)
    I = oracle.importance(Xb)
    I[::37] = 0.0  # dead channels
    c, Is, Ws = bb.awq_prescale(W.cuda(), torch.from_numpy(I).cuda(), Xb.shape[0], j)
    rc, rIs, rWs = oracle.awq_prescale(Wb, I, Xb.shape[0], j)
    assert np.array_equal(f32bits(c), rc.view(np.uint32))
    assert np.array_equal(f32bits(Is), rIs.view(np.uint32))
    assert np.array_equal(u16(Ws), rWs)


def test_prescale_extreme_importance_range():
    """Channel energies spread over 2^-120 .. 2^120 (and exact zeros)."""
    K, tokens = 256, 1000
    rng = np.random.default_rng(3)
    I = (2.0 ** rng.uniform(-120, 120, K)).astype(np.float32)
    I[::11] = 0.0
    W, Wb, _ = _layer(8, K, seed=4)
    for j in (1, 5, 16):
        c, Is, Ws = bb.awq_prescale(W.cuda(), torch.from_numpy(I).cuda(), tokens, j)
        rc, rIs, rWs = oracle.awq_prescale(Wb, I, tokens, j)
        assert np.array_equal(f32bits(c), rc.view(np.uint32))
        assert np.array_equal(f32bits(Is), rIs.view(np.uint32))
        assert np.array_equal(u16(Ws), rWs)


CASES = [(bb.INT4, 128, 16, 48, 512), (bb.INT4, 128, 128, 37, 384), (bb.NVFP4, 16, 16, 40, 256),
         (bb.NVFP4, 16, 8, 24, 208), (bb.NVFP4_GS, 16, 16, 40, 256)]


@pytest.mark.parametrize("fmt,g,S,N,K", CASES)
def test_search_bit_exact(fmt, g, S, N, K):
    iters = 3
    js = [0, 4, 8, 12, 16]
    W, Wb, Xb = _layer(N, K, seed=5 * N + K, dist="normal" if fmt == bb.INT4 else "student_t4")
    I = oracle.importance(Xb)
    cfg = bb.Config(fmt, g, S, iters)
    out = bb.awq_fit(W.cuda(), torch.from_numpy(I).cuda(), Xb.shape[0], cfg, js)
    torch.cuda.synchronize()
    ref = oracle.awq_search(Wb, I, Xb.shape[0], fmt, g, S, iters, js)
    np.testing.assert_allclose(out["err_alpha"].cpu().numpy(), ref["err_alpha"], rtol=RTOL, atol=0)
    assert int(out["best"][0]) == ref["best"]
    assert np.array_equal(f32bits(out["c"]), ref["c"].view(np.uint32))
    assert np.array_equal(out["T_bf16"].cpu().numpy().view(np.uint16), ref["T_bf16"])
    assert np.array_equal(out["codes"].cpu().numpy(), ref["codes"])
    assert np.array_equal(out["scales_tagged"].cpu().numpy().view(ref["scales_tagged"].dtype),
                          ref["scales_tagged"])
    if S != g:
        assert np.array_equal(out["choice_bits"].cpu().numpy(), ref["choice_bits"])
    np.testing.assert_allclose(float(out["err_final"][0]), ref["err_final"], rtol=RTOL)
    if fmt == bb.NVFP4_GS:  # the kept candidate's tensor scale
        assert np.float32(cfg.global_scale.item()) == np.float32(ref["gs"])


def test_search_single_candidate_is_the_plain_fit():
    """One candidate, alpha = 0: the search's output is the plain pipeline's."""
    N, K = 40, 512
    W, Wb, Xb = _layer(N, K, seed=77)
    I = oracle.importance(Xb)
    cfg = bb.Config(bb.INT4, 128, 16, 4)
    Wd, Id = W.cuda(), torch.from_numpy(I).cuda()
    out = bb.awq_fit(Wd, Id, Xb.shape[0], cfg, [0])
    scales, T = bb.init_codebooks(Wd, cfg)
    T, _, _ = bb.fit_layer(Wd, Id, scales, T, cfg)
    plain = bb.pack(Wd, Id, scales, T, cfg)
    torch.cuda.synchronize()
    assert int(out["best"][0]) == 0
    for k in ("T_bf16", "codes", "scales_tagged", "choice_bits"):
        assert torch.equal(out[k], plain[k]), k
    assert float(out["err_final"][0]) == float(plain["err_final"][0])
    assert torch.all(out["c"] == 1.0)


def test_invalid_arguments_launch_nothing():
    W = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    I = torch.ones(64, dtype=torch.float32, device="cuda")
    L = bb.load()
    before = bb.kernel_launches()
    c = torch.empty(64, dtype=torch.float32, device="cuda")
    Ws = torch.empty(4, 64, dtype=torch.int16, device="cuda")
    for j in (-1, 17):
        st = L.aaac_awq_prescale(W.data_ptr(), 4, 64, I.data_ptr(), 10, j, c.data_ptr(),
                                 c.data_ptr(), Ws.data_ptr(), None)
        assert st == 1
    st = L.aaac_awq_prescale(W.data_ptr(), 4, 64, I.data_ptr(), 0, 3, c.data_ptr(),
                             c.data_ptr(), Ws.data_ptr(), None)
    assert st == 2
    cfg = bb.Config(bb.INT4, 64, 64, 1).c()
    js = (ctypes.c_int32 * 18)(*([0] * 18))
    ws = torch.empty(L.aaac_awq_workspace_size(ctypes.byref(cfg), 4, 64), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(64, dtype=torch.uint8, device="cuda")
    e = torch.empty(18, dtype=torch.float64, device="cuda")
    st = L.aaac_awq_fit(W.data_ptr(), 4, 64, I.data_ptr(), 10, ctypes.byref(cfg), js, 18,
                        c.data_ptr(), out.data_ptr(), out.data_ptr(), out.data_ptr(), None,
                        None, e.data_ptr(), None, ws.data_ptr(), ws.numel(), None)
    assert st == 1  # n_alpha > 17
    st = L.aaac_awq_fit(W.data_ptr(), 4, 64, I.data_ptr(), 10, ctypes.byref(cfg), js, 2,
                        c.data_ptr(), out.data_ptr(), out.data_ptr(), out.data_ptr(), None,
                        None, e.data_ptr(), None, ws.data_ptr(), ws.numel() - 256, None)
    assert st == 6  # workspace too small
    torch.cuda.synchronize()
    assert bb.kernel_launches() == before


def test_full_size_gate_prescale():
    """14336 x 4096 with a drawn lognormal importance vector: c and I' over
    all channels, W' on sampled rows, bit-exact."""
    N, K, tokens = 14336, 4096, 262144
    W = synth.make_weight(N, K, 31, device="cuda")
    rng = np.random.default_rng(32)
    I = (np.exp(rng.normal(0, 2, K)) * tokens).astype(np.float32)
    c, Is, Ws = bb.awq_prescale(W, torch.from_numpy(I).cuda(), tokens, 9)
    rows = np.concatenate([[0, 1, N - 1], rng.choice(N, 61, replace=False)])
    Wrows = u16(W[torch.from_numpy(rows).cuda()])
    rc, rIs, rWs = oracle.awq_prescale(Wrows, I, tokens, 9)
    assert np.array_equal(f32bits(c), rc.view(np.uint32))
    assert np.array_equal(f32bits(Is), rIs.view(np.uint32))
    assert np.array_equal(u16(Ws)[rows], rWs)
