"""aaac_fit_layer_fixed_scratch: the fit for callers that cannot allocate.

Some callers cannot call cudaMalloc -- code running where device allocation
is not permitted, or plugins with no access to their host framework's
allocator -- so they cannot hand the library a workspace.  This entry point
runs the same fit with scratch memory the library owns (a fixed-size device
array).  It must give the same results as aaac_fit_layer with a workspace,
call after call, although the array keeps the previous call's contents.

Collected last on purpose (file name), so a run that stops at the first
failure has run every other test already; it also passes on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(N, K, fmt, g, S, iters, seed):
    W, X = synth.small_layer(N, K, seed, T=64, heavy=True)
    W, X = W.cuda(), X.cuda()
    cfg = bb.Config(fmt, g, S, iters)
    I = bb.importance(X)
    scales, T0 = bb.init_codebooks(W, cfg)
    return W, I, scales, T0, cfg


@pytest.mark.parametrize("fmt,g,S", [(bb.INT4, 128, 16), (bb.NVFP4, 16, 16)])
def test_fixed_scratch_matches_workspace_fit(fmt, g, S):
    W, I, scales, T0, cfg = _inputs(384, 1024, fmt, g, S, 6, seed=4242 + S + fmt)
    T_ref, eh_ref, st_ref = bb.fit_layer(W, I, scales, T0.clone(), cfg)
    torch.cuda.synchronize()
    ref_stats = bb.decode_stats(st_ref)
    for call in range(2):  # the second call starts on the first call's leftovers
        T, eh, st = bb.fit_layer_fixed_scratch(W, I, scales, T0.clone(), cfg)
        torch.cuda.synchronize()
        assert torch.equal(T.view(torch.int32), T_ref.view(torch.int32)), call
        np.testing.assert_allclose(eh.cpu().numpy(), eh_ref.cpu().numpy(), rtol=1e-5, atol=0)
        assert bb.decode_stats(st) == ref_stats


def test_fixed_scratch_rejects_layers_past_the_size_limit():
    """Layers with N*K >= 2^31 are rejected before anything is launched (the
    pointers below are never dereferenced: the shape check fails first)."""
    lib = bb.load()
    cfg = bb.Config(bb.INT4, 128, 128, 1).c()
    fake = ctypes.c_void_p(1 << 20)
    st = lib.aaac_fit_layer_fixed_scratch(fake, 1 << 20, 4096, fake, fake, ctypes.byref(cfg),
                                          fake, None, None, None)
    assert st == 2  # AAAC_ERR_SHAPE
    assert b"2^31" in lib.aaac_last_error()
