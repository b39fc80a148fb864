"""The sweep driver on one GPU: a unit written by the sweep equals the oracle
run on the same synthetic inputs (bit-exact tables, codes and tagged scales),
and a second run resumes without recomputing."""
import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200 import sweep, synth

pytestmark = pytest.mark.gpu


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_sweep_unit_matches_oracle_and_resumes(tmp_path):
    wl = synth.WORKLOADS["llama8b-sweep-int4"]
    units = sweep.units_of(wl, layers=range(1), linears=["k_proj", "v_proj"])
    dev = torch.device("cuda", 0)
    tokens, iters = 512, 2
    res = sweep.run_rank(str(tmp_path), units, 0, 1, sweep.gpu_runner(wl, tokens, iters, dev))
    assert res["ran"] == 2 and res["failed"] == 0
    u = units[0]
    X = synth.make_activations(tokens, u.linear.K, synth.seed_of(wl.name, 0, u.linear.x_key, "X"),
                               wl.heavy, device=dev)
    W = synth.make_weight(u.linear.N, u.linear.K, synth.seed_of(wl.name, 0, u.linear.name, "W"),
                          wl.w_dist, device=dev)
    ref = oracle.run_layer(u16(W), u16(X), wl.fmt, wl.g, wl.S, iters)
    with np.load(tmp_path / sweep.load_done(str(tmp_path))[u.uid]["file"]) as z:
        assert np.array_equal(z["T_bf16"].view(np.uint16), ref["T_bf16"])
        assert np.array_equal(z["codes"], ref["codes"])
        assert np.array_equal(z["scales_tagged"].view(np.uint16), ref["scales_tagged"])
    res = sweep.run_rank(str(tmp_path), units, 0, 1, sweep.gpu_runner(wl, tokens, iters, dev))
    assert res["ran"] == 0 and res["skipped"] == 2
