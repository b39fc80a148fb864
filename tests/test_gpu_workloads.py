"""GPU parity at the stated size of every evaluation workload.

"Technical summary: AAAC", section 4: Llama 1B-13B and Qwen 0.5B-32B, NVFP4
g=16 and INT4 g=128.  The synthetic workloads (activation_aware_codebook_b200
/synth.py) stand in for those models; here each runs at its full layer
shapes and its full number of rounds, through the same calls a user makes,
and is compared with the CPU oracle run on the same seeded inputs:

  * Llama-1B-shaped NVFP4 layers (2048x2048, 8192x2048, 2048x8192), 20
    rounds, on the full 16384-token calibration set;
  * one whole layer (its 7 linears) of the 32-layer Llama-8B-shaped INT4
    sweep (S = g = 128), 20 rounds, through the sweep driver, and that
    workload's importance on its full 65536 tokens at sampled columns;
  * the Qwen-32B-shaped NVFP4 gate (27648x5120) and down (5120x27648, the
    widest K of any workload: 54 strips of 512 columns) projections, all 30
    rounds, and their importance on the full 131072 tokens at sampled
    columns.
Where the calibration set is cut for the fit (so that the oracle can redo
every round in minutes), the importance at the full token count is checked
separately, column by column.

The oracle's whole-layer fits take minutes of host time at these sizes.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200 import sweep, synth
from tests.test_gpu_parity import cfg_of, check_against_oracle, u16

pytestmark = pytest.mark.gpu


def _inputs(wl, lin, tokens, layer=0):
    dev = torch.device("cuda", 0)
    W = synth.make_weight(lin.N, lin.K, synth.seed_of(wl.name, layer, lin.name, "W"), wl.w_dist,
                          device=dev)
    X = synth.make_activations(tokens, lin.K, synth.seed_of(wl.name, layer, lin.x_key, "X"),
                               wl.heavy, device=dev)
    return W, X


def _importance_sampled(wl, K, key, tokens, ncols=40):
    """Importance of `tokens` rows of the workload's activations: the fast path
    equals the exact path everywhere and the oracle at sampled columns (the
    heavy channels, both ends, and random ones)."""
    seed = synth.seed_of(wl.name, 0, key, "X")
    X = synth.make_activations(tokens, K, seed, wl.heavy, device="cuda")
    I = bb.importance(X)
    Ie = bb.importance(X, exact=True)
    assert torch.equal(I.view(torch.int32), Ie.view(torch.int32))
    rng = np.random.default_rng(K + tokens)
    heavy = torch.topk(synth.channel_scales(K, seed, wl.heavy, device="cuda"), 5).indices.cpu()
    cols = np.unique(np.concatenate([rng.choice(K, ncols, replace=False), heavy.numpy(),
                                     [0, K - 1]]))
    sub = u16(X[:, torch.from_numpy(cols).cuda()].contiguous())
    ref = oracle.importance(sub)
    assert np.array_equal(I.cpu().numpy()[cols].view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("idx", [0, 1, 2])
def test_llama1b_nvfp4_layers_full_size(idx):
    wl = synth.WORKLOADS["llama1b-nvfp4"]
    lin = wl.linears[idx]
    W, X = _inputs(wl, lin, wl.tokens)
    cfg = cfg_of(wl.fmt, wl.g, wl.S, wl.iters)
    out = bb.run_layer(W, X, cfg)
    ref = oracle.run_layer(u16(W), u16(X), wl.fmt, wl.g, wl.S, wl.iters)
    check_against_oracle(out, ref, cfg, label=lin.name)


def test_llama8b_sweep_one_whole_layer(tmp_path):
    """Layer 0's seven linears through the sweep driver, 20 rounds each; every
    unit's stored tables, codes, tagged scales, statistics and objectives
    against the oracle's run of the same unit."""
    wl = synth.WORKLOADS["llama8b-sweep-int4"]
    units = sweep.units_of(wl, layers=range(1))
    assert len(units) == 7
    dev = torch.device("cuda", 0)
    tokens = 4096  # the importance at the full 65536 tokens is checked below
    res = sweep.run_rank(str(tmp_path), units, 0, 1, sweep.gpu_runner(wl, tokens, wl.iters, dev))
    assert res["ran"] == 7 and res["failed"] == 0
    done = sweep.load_done(str(tmp_path))
    I_cache = {}
    for u in units:
        W, X = _inputs(wl, u.linear, tokens)
        Wb = u16(W)
        if u.linear.x_key not in I_cache:
            I_cache[u.linear.x_key] = oracle.importance(u16(X))
        I = I_cache[u.linear.x_key]
        scl, T0, gs = oracle.init_codebooks(Wb, wl.fmt, wl.g, with_gs=True)
        T, err, st = oracle.fit(Wb, I, scl, T0, wl.fmt, wl.g, wl.S, wl.iters)
        ref = oracle.pack(Wb, I, scl, T, wl.fmt, wl.g, wl.S)
        with np.load(tmp_path / done[u.uid]["file"]) as z:
            assert np.array_equal(z["T"].view(np.uint32), T.view(np.uint32)), u.uid
            assert np.array_equal(z["T_bf16"].view(np.uint16), ref["T_bf16"]), u.uid
            assert np.array_equal(z["codes"], ref["codes"]), u.uid
            assert np.array_equal(z["scales_tagged"].view(np.uint16), ref["scales_tagged"]), u.uid
            near, t1, empty, dead, exact, L = (int(v) for v in z["stats"])
            assert (near, t1, empty, dead, L) == (st.near_ties, st.groups_t1, st.empty_cells,
                                                  st.dead_groups, st.L), u.uid
            assert exact >= near
            np.testing.assert_allclose(z["err_hist"], err, rtol=1e-5, atol=0)
            np.testing.assert_allclose(float(z["err_final"][0]), ref["err_final"], rtol=1e-5)
        del W, X


@pytest.mark.parametrize("K,key", [(4096, "attn_in"), (14336, "mlp_act")])
def test_llama8b_sweep_importance_full_tokens(K, key):
    wl = synth.WORKLOADS["llama8b-sweep-int4"]
    _importance_sampled(wl, K, key, wl.tokens)


@pytest.mark.parametrize("idx", [0, 2])
def test_qwen32b_nvfp4_all_rounds(idx):
    """gate (27648x5120) and down (5120x27648) for all 30 rounds."""
    wl = synth.WORKLOADS["qwen32b-nvfp4"]
    lin = wl.linears[idx]
    W, X = _inputs(wl, lin, 2048)
    cfg = cfg_of(wl.fmt, wl.g, wl.S, wl.iters)
    out = bb.run_layer(W, X, cfg)
    ref = oracle.run_layer(u16(W), u16(X), wl.fmt, wl.g, wl.S, wl.iters)
    check_against_oracle(out, ref, cfg, label=lin.name)


@pytest.mark.parametrize("K,key", [(5120, "h"), (27648, "a")])
def test_qwen32b_importance_full_tokens(K, key):
    wl = synth.WORKLOADS["qwen32b-nvfp4"]
    _importance_sampled(wl, K, key, wl.tokens)
