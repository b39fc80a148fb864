"""The near-tie count on the GPU, against the oracle.

"Technical summary: AAAC", section 2, core mechanism 2 (the choice by the
lower activation-weighted error); the parity contract counts groups whose two
errors differ by less than 1e-6 of the larger one.  The hand-built layer of
tests/test_oracle_neartie.py (errors known exactly, ties just inside and just
outside the band) goes through aaac_fit_layer with both books frozen; the
count, the T1 groups and the objective must be the oracle's, for the two-book
fit and for SINGLE_CODEBOOK.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import binding as bb
from tests.test_oracle_neartie import GROUPS, _layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("single", [False, True])
def test_near_ties_of_hand_built_groups(single):
    W, I, T = _layer()
    flags = bb.FREEZE_T0 | bb.FREEZE_T1 | (bb.SINGLE_CODEBOOK if single else 0)
    cfg = bb.Config(bb.INT4, 16, 16, 2, flags)
    Wd = torch.from_numpy(W.view(np.int16)).cuda()
    Id = torch.from_numpy(I).cuda()
    scales, _ = bb.init_codebooks(Wd, cfg)
    Td = torch.from_numpy(T.copy()).cuda()
    T_out, eh, st = bb.fit_layer(Wd, Id, scales, Td, cfg)
    torch.cuda.synchronize()
    s = bb.decode_stats(st)
    ref_scl, _ = oracle.init_codebooks(W, oracle.INT4, 16)
    _, err, rst = oracle.fit(W, I, ref_scl, T, oracle.INT4, 16, 16, 2, flags)
    assert s["near_ties"] == rst.near_ties == sum(1 for g in GROUPS if g[2])
    assert s["groups_t1"] == rst.groups_t1
    assert s["exact_groups"] >= 2 * s["near_ties"]  # each round decides them exactly
    np.testing.assert_allclose(eh.cpu().numpy(), err, rtol=1e-9, atol=0)
    assert np.array_equal(T_out.cpu().numpy(), T)
