"""GPU parity: libaaac (through the C ABI) against the CPU oracle, element by
element, on seeded synthetic inputs.

Bar (AAAC fit contract): importance, scales, initial codebooks, fitted
codebooks, codes, choice bits and tagged scales bit-exact; err_hist and
err_final within 1e-5 relative (the GPU sums them in a different order and
takes clear-cut codebook choices from fp32 sums).
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
    a = t.detach().cpu().contiguous().numpy()
    return a.view(np.uint32) if a.dtype == np.float32 else a


def cfg_of(fmt, g, S, iters, flags=0):
    return bb.Config(fmt, g, S, iters, flags)


def layer(N, K, seed, T=64, heavy=True, dist="normal"):
    W, X = synth.small_layer(N, K, seed, T=T, heavy=heavy, dist=dist)
    return W.cuda(), X.cuda()


# --------------------------------------------------------------------------
# importance
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T,K", [(128, 512), (1000, 520), (7, 8), (3000, 4096)])
def test_importance_bit_exact(T, K):
    X = synth.make_activations(T, K, seed=T + K, heavy=True).cuda()
    I = bb.importance(X)
    ref = oracle.importance(u16(X))
    assert np.array_equal(npbits(I), ref.view(np.uint32))
    Ie = bb.importance(X, exact=True)
    assert np.array_equal(npbits(Ie), ref.view(np.uint32))


def test_importance_accumulate_strided_and_boundary():
    X = synth.make_activations(300, 264, seed=5, heavy=False)
    wide = torch.zeros(300, 272, dtype=torch.bfloat16)
    wide[:, :264] = X
    wide = wide.cuda()
    I = bb.importance(wide[:120], ncols=264)
    I = bb.importance(wide[120:], I=I, accumulate=True, ncols=264)
    Xb = u16(X)
    ref = oracle.importance(Xb[120:], I_in=oracle.importance(Xb[:120]))
    assert np.array_equal(npbits(I), ref.view(np.uint32))
    # columns whose fp64 sum sits on an fp32 rounding boundary
    cols = [[4096.0, 1.0, 2.0 ** -60, 0.0], [4096.0, 1.0, 0.0, 0.0],
            [4096.0, 1.0, -(2.0 ** -60), 2.0 ** -61], [1e-39, -1e-39, 2.0 ** -130, 0.0],
            [2.0 ** 64, 0.0, 0.0, 0.0], [3.0, 5.0, 7.0, 11.0], [0, 0, 0, 0], [1, 1, 1, 1]]
    Xc = torch.tensor(cols, dtype=torch.float32).t().contiguous().to(torch.bfloat16)
    Ig = bb.importance(Xc.cuda())
    assert np.array_equal(npbits(Ig), oracle.importance(u16(Xc)).view(np.uint32))
    assert float(Ig[0]) == 2.0 ** 24 + 2 and float(Ig[1]) == 2.0 ** 24


# --------------------------------------------------------------------------
# scales, init, fit, pack
# --------------------------------------------------------------------------
CASES = [(bb.INT4, 128, 128, 256, 512), (bb.INT4, 128, 16, 37, 640), (bb.NVFP4, 16, 16, 64, 512),
         (bb.INT4, 32, 8, 48, 256), (bb.NVFP4, 16, 16, 33, 1040), (bb.NVFP4, 16, 8, 40, 528),
         (bb.NVFP4_GS, 16, 16, 64, 512), (bb.NVFP4_GS, 16, 8, 33, 1040)]


@pytest.mark.parametrize("fmt,g,S,N,K", CASES)
def test_init_bit_exact(fmt, g, S, N, K):
    W, _ = layer(N, K, seed=N * K + g)
    cfg = cfg_of(fmt, g, S, 0)
    scl, T = bb.init_codebooks(W, cfg)
    rscl, rT, rgs = oracle.init_codebooks(u16(W), fmt, g, with_gs=True)
    assert np.array_equal(scl.cpu().numpy().view(rscl.dtype), rscl)
    assert np.array_equal(npbits(T), rT.view(np.uint32))
    if fmt == bb.NVFP4_GS:
        assert np.float32(cfg.global_scale.item()) == np.float32(rgs)


@pytest.mark.parametrize("fmt,g,S,N,K", CASES)
@pytest.mark.parametrize("iters", [1, 6])
def test_fit_and_pack_bit_exact(fmt, g, S, N, K, iters):
    W, X = layer(N, K, seed=3 * N + K + iters, dist="normal" if fmt == bb.INT4 else "student_t4")
    cfg = cfg_of(fmt, g, S, iters)
    out = bb.run_layer(W, X, cfg)
    ref = oracle.run_layer(u16(W), u16(X), fmt, g, S, iters)
    check_against_oracle(out, ref, cfg)


def check_against_oracle(out, ref, cfg, label=""):
    torch.cuda.synchronize()
    assert np.array_equal(npbits(out["I"]), ref["I"].view(np.uint32)), label
    assert np.array_equal(out["scales"].cpu().numpy().view(ref["scales"].dtype), ref["scales"])
    if cfg.fmt == bb.NVFP4_GS:
        assert np.float32(out["global_scale"].item()) == np.float32(ref["gs"]), label
    if "T_init" in out:  # the bench's block keeps no copy of the initial tables
        assert np.array_equal(npbits(out["T_init"]), ref["T_init"].view(np.uint32)), label
    T, rT = out["T"].cpu().numpy(), ref["T"]
    assert np.array_equal(T.view(np.uint32), rT.view(np.uint32)), (label, T, rT)
    st = bb.decode_stats(out["stats"])
    assert st["L"] == ref["stats"].L
    if cfg.iters:
        assert st["groups_t1"] == ref["stats"].groups_t1
        assert st["empty_cells"] == ref["stats"].empty_cells
        assert st["dead_groups"] == ref["stats"].dead_groups
        # near ties (reading R13) of the last round; each was decided by the
        # exact fp64 rule, which the exact-decision count (all rounds) includes
        assert st["near_ties"] == ref["stats"].near_ties, label
        assert st["exact_groups"] >= st["near_ties"], label
        eh = out["err_hist"].cpu().numpy()
        np.testing.assert_allclose(eh, ref["err_hist"], rtol=RTOL, atol=0)
    assert np.array_equal(out["T_bf16"].cpu().numpy().view(np.uint16), ref["T_bf16"])
    assert np.array_equal(out["codes"].cpu().numpy(), ref["codes"]), label
    assert np.array_equal(out["scales_tagged"].cpu().numpy().view(ref["scales_tagged"].dtype),
                          ref["scales_tagged"])
    if cfg.S != cfg.g:
        assert np.array_equal(out["choice_bits"].cpu().numpy(), ref["choice_bits"])
    np.testing.assert_allclose(float(out["err_final"][0]), ref["err_final"], rtol=RTOL)


@pytest.mark.parametrize("fmt,g,S,N,K", [(bb.INT4, 128, 16, 1024, 4096),
                                         (bb.NVFP4_GS, 16, 16, 2048, 2048),
                                         (bb.INT4, 128, 128, 14336, 4096)])
def test_concurrent_grid_same_results(fmt, g, S, N, K):
    """AAAC_CONCURRENT only resizes the fit and pack grids: every output is
    the full-grid call's, bit for bit."""
    W, X = layer(N, K, seed=N + K, T=256, dist="normal" if fmt == bb.INT4 else "student_t4")
    ref = bb.run_layer(W, X, cfg_of(fmt, g, S, 4))
    out = bb.run_layer(W, X, cfg_of(fmt, g, S, 4, flags=bb.CONCURRENT))
    torch.cuda.synchronize()
    for k in ("I", "scales", "T_init", "T", "err_hist", "stats", "T_bf16", "codes",
              "scales_tagged", "err_final") + (("choice_bits",) if S != g else ()):
        assert torch.equal(out[k], ref[k]), k


def test_many_strips_single_counter():
    """K = 131584 (257 strips of 512 columns): past the per-strip counters the
    pass hands out fixed-size items from one counter; with 48 rows there are
    more items than warps in a full wave, so some are claimed."""
    N, K, iters = 48, 257 * 512, 3
    W, X = layer(N, K, seed=257, T=32)
    cfg = cfg_of(bb.INT4, 128, 16, iters)
    out = bb.run_layer(W, X, cfg)
    ref = oracle.run_layer(u16(W), u16(X), bb.INT4, 128, 16, iters)
    check_against_oracle(out, ref, cfg, label="257 strips")


@pytest.mark.parametrize("fmt,g,S,N,K", [(bb.INT4, 128, 128, 1, 128), (bb.NVFP4, 16, 16, 1, 16),
                                         (bb.NVFP4, 16, 8, 3, 16), (bb.INT4, 16, 8, 5, 48),
                                         (bb.NVFP4_GS, 16, 16, 2, 32)])
@pytest.mark.parametrize("iters", [0, 3])
def test_tiny_layers(fmt, g, S, N, K, iters):
    """One row, one scale group, a 16-weight layer, and zero rounds (the pack
    straight after the init): every output bit-exact against the oracle."""
    W, X = layer(N, K, seed=7 * N + K + iters, T=32,
                 dist="normal" if fmt == bb.INT4 else "student_t4")
    cfg = cfg_of(fmt, g, S, iters)
    out = bb.run_layer(W, X, cfg)
    ref = oracle.run_layer(u16(W), u16(X), fmt, g, S, iters)
    check_against_oracle(out, ref, cfg, label=f"{N}x{K}")


def test_single_256x512_int4_workload():
    """The 256x512 INT4 g=128 S=128 layer, X[128, 512], 10 iterations, seed 0."""
    wl = synth.WORKLOADS["single-256x512-int4"]
    lin = wl.linears[0]
    W = synth.make_weight(lin.N, lin.K, synth.seed_of(wl.name, 0, lin.name, "W"))
    X = synth.make_activations(wl.tokens, lin.K, synth.seed_of(wl.name, 0, lin.name, "X"),
                               wl.heavy)
    cfg = cfg_of(wl.fmt, wl.g, wl.S, wl.iters)
    out = bb.run_layer(W.cuda(), X.cuda(), cfg)
    ref = oracle.run_layer(u16(W), u16(X), wl.fmt, wl.g, wl.S, wl.iters)
    check_against_oracle(out, ref, cfg)
    eh = out["err_hist"].cpu().numpy()
    assert np.all(eh[1:] <= eh[:-1] * (1 + 1e-6))


# --------------------------------------------------------------------------
# degenerate inputs
# --------------------------------------------------------------------------
def test_dead_groups_constant_weights_and_duplicates():
    N, K, g = 40, 256, 16
    W = synth.make_weight(N, K, seed=90)
    W[0] = 0                      # every group of row 0 has s = 0
    W[1, :64] = 1e-4              # NVFP4: scale underflows to 0
    W[2:10] = 0.5                 # constant groups: heavy duplicate u values
    X = synth.make_activations(32, K, seed=91, heavy=True)
    X[:, 10:20] = 0               # columns with zero importance
    for fmt, S in ((bb.NVFP4, 16), (bb.INT4, 16), (bb.NVFP4_GS, 16)):
        cfg = cfg_of(fmt, g, S, 5)
        out = bb.run_layer(W.cuda(), X.cuda(), cfg)
        ref = oracle.run_layer(u16(W), u16(X), fmt, g, S, 5)
        check_against_oracle(out, ref, cfg, label=f"fmt{fmt}")
        assert bb.decode_stats(out["stats"])["dead_groups"] > 0


@pytest.mark.parametrize("sigma", [1e-3, 0.0])
def test_tensor_scale_small_and_zero_weights(sigma):
    """NVFP4 with a per-tensor scale on weights whose group maxima are E4M3
    subnormals without it (about 2e-3), and on an all-zero tensor (gs = 0,
    every group dead)."""
    N, K = 48, 512
    W = (synth.make_weight(N, K, seed=95).float() * (sigma / 0.02)).to(torch.bfloat16)
    X = synth.make_activations(64, K, seed=96, heavy=True)
    cfg = cfg_of(bb.NVFP4_GS, 16, 16, 4)
    out = bb.run_layer(W.cuda(), X.cuda(), cfg)
    ref = oracle.run_layer(u16(W), u16(X), bb.NVFP4_GS, 16, 16, 4)
    check_against_oracle(out, ref, cfg)
    if sigma == 0.0:
        assert float(out["global_scale"][0]) == 0.0
        assert bb.decode_stats(out["stats"])["dead_groups"] == N * K // 16


def test_all_equal_weights():
    W = torch.full((16, 256), 0.25, dtype=torch.bfloat16)
    X = synth.make_activations(16, 256, seed=92, heavy=False)
    cfg = cfg_of(bb.INT4, 128, 128, 3)
    out = bb.run_layer(W.cuda(), X.cuda(), cfg)
    ref = oracle.run_layer(u16(W), u16(X), bb.INT4, 128, 128, 3)
    check_against_oracle(out, ref, cfg)


@pytest.mark.parametrize("flags", [bb.FREEZE_T0 | bb.FREEZE_T1, bb.SINGLE_CODEBOOK, bb.FREEZE_T1])
def test_flags_rtn_single_frozen(flags):
    N, K, g = 64, 512, 128
    W, X = layer(N, K, seed=93 + flags)
    cfg = cfg_of(bb.INT4, g, 16, 4, flags)
    I = bb.importance(X)
    scl, _ = bb.init_codebooks(W, cfg)
    grid = torch.arange(-8, 8, dtype=torch.float32)
    T0 = torch.stack([grid, grid + 0.5]).cuda()
    T, eh, st = bb.fit_layer(W, I, scl, T0.clone(), cfg)
    out = bb.pack(W, I, scl, T, cfg)
    Wb, Ib, sb = u16(W), I.cpu().numpy(), scl.cpu().numpy()
    rT, reh, rst = oracle.fit(Wb, Ib, sb, T0.cpu().numpy(), bb.INT4, g, 16, 4, flags)
    assert np.array_equal(npbits(T), rT.view(np.uint32))
    np.testing.assert_allclose(eh.cpu().numpy()[:4], reh, rtol=RTOL)
    rp = oracle.pack(Wb, Ib, sb, rT, bb.INT4, g, 16, flags)
    assert np.array_equal(out["codes"].cpu().numpy(), rp["codes"])
    assert np.array_equal(out["choice_bits"].cpu().numpy(), rp["choice_bits"])
    if flags & bb.SINGLE_CODEBOOK:
        assert not out["choice_bits"].any()


def test_crowded_buckets_duplicates_and_signed_zeros():
    """Codebooks with entries 0.02 apart (several midpoint thresholds inside
    one lookup bucket: the exact binary search takes over), equal entries
    (one cell), and -0 / +0 (equal values, one cell)."""
    N, K, g = 96, 512, 128
    W, X = layer(N, K, seed=97)
    cfg = cfg_of(bb.INT4, g, 16, 2)
    I = bb.importance(X)
    scl, _ = bb.init_codebooks(W, cfg)
    b0 = [-3, -2, -1, 0.50, 0.52, 0.54, 0.56, 1, 2, 3, 4, 5, 6, -4, -5, 7]
    b1 = [-7.5, -6.5, -0.0, 0.0, 0.031, 0.033, 0.035, 1.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5, -1.5, -2.5]
    T0 = torch.tensor([b0, b1], dtype=torch.float32).cuda()
    for iters in (1, 2):
        c = cfg_of(bb.INT4, g, 16, iters)
        T, eh, st = bb.fit_layer(W, I, scl, T0.clone(), c)
        Wb, Ib, sb = u16(W), I.cpu().numpy(), scl.cpu().numpy()
        rT, reh, rst = oracle.fit(Wb, Ib, sb, T0.cpu().numpy(), bb.INT4, g, 16, iters)
        assert np.array_equal(npbits(T), rT.view(np.uint32))
    out = bb.pack(W, I, scl, T0, cfg)
    rp = oracle.pack(u16(W), I.cpu().numpy(), scl.cpu().numpy(), T0.cpu().numpy(), bb.INT4, g, 16)
    assert np.array_equal(out["codes"].cpu().numpy(), rp["codes"])
    assert np.array_equal(out["choice_bits"].cpu().numpy(), rp["choice_bits"])


def test_deterministic_bits():
    W, X = layer(512, 1024, seed=95)
    cfg = cfg_of(bb.INT4, 128, 16, 8)
    a = bb.run_layer(W, X, cfg)
    b = bb.run_layer(W, X, cfg)
    for k in ("I", "T", "codes", "scales_tagged", "choice_bits", "err_final", "err_hist"):
        assert torch.equal(a[k].view(torch.uint8), b[k].view(torch.uint8)), k


# --------------------------------------------------------------------------
# full-size layers (the oracle still finishes in seconds on these)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name,idx,iters", [("llama1b-nvfp4", 0, 20), ("llama8b-int4-s16", 1, 20)])
def test_full_size_layer(name, idx, iters):
    wl = synth.WORKLOADS[name]
    lin = wl.linears[idx]
    W = synth.make_weight(lin.N, lin.K, synth.seed_of(wl.name, 0, lin.name, "W"), wl.w_dist)
    tokens = 4096  # importance parity at full token count is tested separately
    X = synth.make_activations(tokens, lin.K, synth.seed_of(wl.name, 0, lin.x_key, "X"), wl.heavy)
    cfg = cfg_of(wl.fmt, wl.g, wl.S, iters)
    out = bb.run_layer(W.cuda(), X.cuda(), cfg)
    ref = oracle.run_layer(u16(W), u16(X), wl.fmt, wl.g, wl.S, iters)
    check_against_oracle(out, ref, cfg, label=name)


# --------------------------------------------------------------------------
# full bench sizes: importance on 262144 tokens (sampled columns), and the
# largest (Qwen-32B-shaped, NVFP4) layer for a few rounds
# --------------------------------------------------------------------------
@pytest.mark.parametrize("K", [4096, 14336])
def test_importance_full_tokens_sampled_columns(K):
    wl = synth.WORKLOADS["llama8b-int4-s16"]
    X = synth.make_activations(wl.tokens, K, synth.seed_of(wl.name, 0, f"probe{K}", "X"), wl.heavy,
                               device="cuda")
    I = bb.importance(X)
    Ie = bb.importance(X, exact=True)
    rng = np.random.default_rng(K)
    cols = np.sort(rng.choice(K, 48, replace=False))
    heavy = torch.topk(synth.channel_scales(K, synth.seed_of(wl.name, 0, f"probe{K}", "X") ^ 0,
                                            wl.heavy, device="cuda"), 3).indices.cpu().numpy()
    cols = np.unique(np.concatenate([cols, heavy, [0, K - 1]]))
    sub = u16(X[:, torch.from_numpy(cols).cuda()].contiguous())
    ref = oracle.importance(sub)
    got = I.cpu().numpy()[cols]
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert torch.equal(I.view(torch.int32), Ie.view(torch.int32))  # fast path == exact path
    del X


def test_qwen32b_nvfp4_full_layer_few_rounds():
    wl = synth.WORKLOADS["qwen32b-nvfp4"]
    lin = wl.linears[0]  # gate 27648x5120, Student-t weights
    W = synth.make_weight(lin.N, lin.K, synth.seed_of(wl.name, 0, lin.name, "W"), wl.w_dist,
                          device="cuda")
    X = synth.make_activations(2048, lin.K, synth.seed_of(wl.name, 0, lin.x_key, "X"), wl.heavy,
                               device="cuda")
    cfg = cfg_of(wl.fmt, wl.g, wl.S, 2)
    out = bb.run_layer(W, X, cfg)
    ref = oracle.run_layer(u16(W), u16(X), wl.fmt, wl.g, wl.S, 2)
    check_against_oracle(out, ref, cfg, label="qwen32b gate")



def test_bench_launch_configuration_full_size():
    """The bench step as bench.py launches it: the Llama-3-8B-shaped block,
    every linear on its own stream with its own workspace (biggest first) and
    each activation set's importance on its own stream, all in flight at once.
    Layer sizes are the bench's; the calibration set is cut to 4096 tokens so
    that the oracle can redo the whole 20-round fit of gate_proj (58.7M
    weights) and of k_proj on the CPU."""
    import bench
    wl = synth.WORKLOADS["llama8b-int4-s16"]
    dev = torch.device("cuda", 0)
    Xs, Ws = bench.build_block(wl, 0, 4096, dev)
    blk = bench.Block(wl, Xs, Ws, dev)
    blk.step()
    torch.cuda.synchronize()
    cfg = cfg_of(wl.fmt, wl.g, wl.S, wl.iters)
    for name in ("gate_proj", "k_proj"):
        lin = next(l for l in wl.linears if l.name == name)
        ref = oracle.run_layer(u16(Ws[name]), u16(Xs[lin.x_key]), wl.fmt, wl.g, wl.S, wl.iters)
        out = dict(blk.out[name], I=blk.I[lin.x_key], scales=blk.scales[name], T=blk.T[name],
                   stats=blk.st[name], err_hist=blk.eh[name])
        check_against_oracle(out, ref, cfg, label=name)
    assert bb.device_timeouts() == 0
