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


_SECOND_CONTEXT = r"""
import ctypes, sys
import numpy as np
import torch
from cuda.bindings import driver as cu
from activation_aware_codebook_b200 import binding as bb, synth

def ok(r):
    err = r[0] if isinstance(r, tuple) else r
    assert err == cu.CUresult.CUDA_SUCCESS, err
    return r[1] if isinstance(r, tuple) and len(r) > 1 else None

N, K, iters = 96, 512, 4
W, X = synth.small_layer(N, K, 21, T=64, heavy=True)
W, X = W.cuda(), X.cuda()
cfg = bb.Config(bb.INT4, 128, 16, iters)
I = bb.importance(X)
scales, T0 = bb.init_codebooks(W, cfg)
T_ref, eh_ref, _ = bb.fit_layer_fixed_scratch(W, I, scales, T0.clone(), cfg)
torch.cuda.synchronize()
host = {"W": W.view(torch.int16).cpu().numpy(), "I": I.cpu().numpy(),
        "s": scales.view(torch.int16).cpu().numpy(), "T": T0.cpu().numpy()}

# a second context on the same device, current to this thread
ok(cu.cuInit(0))
dev = ok(cu.cuDeviceGet(0))
ctx = ok(cu.cuCtxCreate(0, dev))
bufs = {}
for k, a in host.items():
    a = np.ascontiguousarray(a)
    d = ok(cu.cuMemAlloc(a.nbytes))
    ok(cu.cuMemcpyHtoD(d, a.ctypes.data, a.nbytes))
    bufs[k] = d
eh = ok(cu.cuMemAlloc(8 * iters))
st = ok(cu.cuMemAlloc(bb.STATS_BYTES))
c = cfg.c()
lib = bb.load()
p = lambda d: ctypes.c_void_p(int(d))
rc = lib.aaac_fit_layer_fixed_scratch(p(bufs["W"]), N, K, p(bufs["I"]), p(bufs["s"]),
                                      ctypes.byref(c), p(bufs["T"]), p(eh), p(st), None)
assert rc == 0, lib.aaac_last_error()
ok(cu.cuCtxSynchronize())
T2 = np.empty_like(host["T"])
ok(cu.cuMemcpyDtoH(T2.ctypes.data, bufs["T"], T2.nbytes))
eh2 = np.empty(iters, dtype=np.float64)
ok(cu.cuMemcpyDtoH(eh2.ctypes.data, eh, eh2.nbytes))
for d in list(bufs.values()) + [eh, st]:
    ok(cu.cuMemFree(d))
ok(cu.cuCtxDestroy(ctx))
assert np.array_equal(T2.view(np.uint32), T_ref.cpu().numpy().view(np.uint32))
assert np.array_equal(eh2, eh_ref.cpu().numpy())
# back on the primary context: the same fit again
T3, _, _ = bb.fit_layer_fixed_scratch(W, I, scales, T0.clone(), cfg)
torch.cuda.synchronize()
assert torch.equal(T3.view(torch.int32), T_ref.view(torch.int32))
print("SECOND CONTEXT OK")
"""


def test_fixed_scratch_in_a_second_context():
    """The library-owned scratch is looked up again when another context on
    the same device is current (a second context loads the library's module
    anew, and the array gets another address there): the fit in a context
    made with cuCtxCreate equals the primary context's, and the primary
    context's next call is right too.  Run in a child process, so that the
    extra context does not outlive the test."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _SECOND_CONTEXT], cwd=root,
                         env=dict(os.environ, PYTHONPATH=root), capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    assert "SECOND CONTEXT OK" in res.stdout
