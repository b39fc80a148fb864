"""The whole per-layer path captured once in a CUDA graph and replayed.

Every libaaac call works on caller-owned buffers and a caller-owned workspace,
never allocates and never waits on the host, and the fit rounds use
programmatic dependent launches; so importance -> init -> fit -> pack (and the
linear that consumes the packed layer) can be captured and replayed on new
inputs copied into the same buffers.  Replays must give the oracle's results
bit for bit, like eager calls.
"""
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


def npbits(t):
    return t.detach().cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("fmt,g,S", [(bb.INT4, 128, 16), (bb.NVFP4_GS, 16, 16), (bb.NVFP4, 16, 8)])
def test_layer_path_in_a_cuda_graph(fmt, g, S):
    N, K, T, iters = 96, 768, 64, 4
    dev = torch.device("cuda")
    cfg = bb.Config(fmt, g, S, iters)
    cfg.ensure_global_scale(dev)
    W = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    X = torch.empty(T, K, dtype=torch.bfloat16, device=dev)
    ws = bb.workspace(cfg, N, K, T, dev)
    I = torch.empty(K, dtype=torch.float32, device=dev)
    sdt = torch.int16 if fmt == bb.INT4 else torch.uint8
    scales = torch.empty(N, K // g, dtype=sdt, device=dev)
    Tt = torch.empty(2, 16, dtype=torch.float32, device=dev)
    eh = torch.zeros(iters, dtype=torch.float64, device=dev)
    st = torch.zeros(bb.STATS_BYTES, dtype=torch.uint8, device=dev)
    out = dict(T_bf16=torch.zeros(2, 16, dtype=torch.int16, device=dev),
               codes=torch.empty(N, K // 2, dtype=torch.uint8, device=dev),
               scales_tagged=torch.empty(N, K // g, dtype=sdt, device=dev),
               choice_bits=(torch.empty(N, (K // S + 7) // 8, dtype=torch.uint8, device=dev)
                            if S != g else None),
               err_final=torch.zeros(1, dtype=torch.float64, device=dev))
    x1 = torch.empty(1, K, dtype=torch.bfloat16, device=dev)
    Y = torch.empty(1, N, dtype=torch.float32, device=dev)
    x16 = torch.empty(16, K, dtype=torch.bfloat16, device=dev)
    Y16 = torch.empty(16, N, dtype=torch.float32, device=dev)

    def path():
        bb.importance(X, I=I, ws=ws)
        bb.init_codebooks(W, cfg, ws=ws, scales=scales, T=Tt)
        bb.fit_layer(W, I, scales, Tt, cfg, ws=ws, err_hist=eh, stats=st)
        bb.pack(W, I, scales, Tt, cfg, ws=ws, out=out)
        bb.linear(x1, out, cfg, N, K, out=Y)     # CUDA-core GEMV
        bb.linear(x16, out, cfg, N, K, out=Y16)  # tcgen05 GEMM

    def load(seed):
        Wn, Xn = synth.small_layer(N, K, seed, T=T, heavy=True,
                                   dist="normal" if fmt == bb.INT4 else "student_t4")
        W.copy_(Wn)
        X.copy_(Xn)
        x1.copy_(synth.make_activations(1, K, seed + 1000, True))
        x16.copy_(synth.make_activations(16, K, seed + 2000, True))
        return u16(Wn), u16(Xn)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        load(1)
        path()  # warm-up outside the capture (kernel attributes, lazy loading)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    launches0 = bb.kernel_launches()
    with torch.cuda.graph(graph):
        path()
    captured = bb.kernel_launches() - launches0
    assert captured > iters

    for seed in (2, 3):
        Wb, Xb = load(seed)
        torch.cuda.synchronize()
        before = bb.kernel_launches()
        graph.replay()
        torch.cuda.synchronize()
        assert bb.kernel_launches() == before  # replays launch from the graph, not the host
        ref = oracle.run_layer(Wb, Xb, fmt, g, S, iters)
        assert np.array_equal(npbits(I), ref["I"].view(np.uint32))
        assert np.array_equal(scales.cpu().numpy().view(ref["scales"].dtype), ref["scales"])
        assert np.array_equal(npbits(Tt), ref["T"].view(np.uint32))
        np.testing.assert_allclose(eh.cpu().numpy(), ref["err_hist"], rtol=RTOL)
        assert np.array_equal(out["codes"].cpu().numpy(), ref["codes"])
        if S != g:
            assert np.array_equal(out["choice_bits"].cpu().numpy(), ref["choice_bits"])
        assert np.array_equal(u16(out["T_bf16"]), ref["T_bf16"])
        if fmt == bb.NVFP4_GS:
            assert np.float32(cfg.global_scale.item()) == np.float32(ref["gs"])
        Wh = oracle.dequant_bf16(ref["codes"], ref["scales_tagged"], ref["choice_bits"],
                                 ref["T_bf16"], N, K, fmt, g, S, ref["gs"])
        ww = np.abs((np.asarray(Wh, dtype=np.uint32) << 16).view(np.float32).astype(np.float64))
        for xin, yout in ((x1, Y), (x16, Y16)):
            yref = oracle.linear(u16(xin), Wh)
            xw = np.abs((np.asarray(u16(xin), dtype=np.uint32) << 16).view(np.float32)
                        .astype(np.float64))
            bound = K * 2.0 ** -24 * (xw @ ww.T) + 1e-30
            assert np.all(np.abs(yout.cpu().numpy().astype(np.float64) - yref) <= bound)
        assert bb.device_timeouts() == 0
    del graph
