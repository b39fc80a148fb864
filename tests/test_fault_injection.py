"""Host-side fault injection (no GPU needed): an armed fault makes the next
call that would launch work return its error after the argument checks,
before anything reaches a GPU, with every output untouched; it fires once.

The buffers below are host memory: the calls only check pointers for
alignment before the point where the fault fires, so nothing dereferences
them as device memory and their bytes must come back unchanged.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest

from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200.csrc import build as cbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return bb.load()


def _host(nbytes, fill):
    a = np.full(nbytes + 64, fill, dtype=np.uint8)
    off = (-a.ctypes.data) % 16  # 16-byte aligned view
    return a[off:off + nbytes]


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _fit_call(lib, bufs):
    N, K = 64, 256
    cfg = bb.Config(bb.INT4, 128, 16, 3).c()
    return lib.aaac_fit_layer(_ptr(bufs["W"]), N, K, _ptr(bufs["I"]), _ptr(bufs["scales"]),
                              ctypes.byref(cfg), _ptr(bufs["T"]), _ptr(bufs["eh"]),
                              _ptr(bufs["st"]), _ptr(bufs["ws"]), bufs["ws"].size, None)


def _buffers(lib):
    N, K = 64, 256
    cfg = bb.Config(bb.INT4, 128, 16, 3)
    ws = lib.aaac_workspace_size(ctypes.byref(cfg.c()), N, K, 0)
    return {"W": _host(N * K * 2, 3), "I": _host(K * 4, 5), "scales": _host(N * 2 * 2, 7),
            "T": _host(128, 9), "eh": _host(3 * 8, 11), "st": _host(48, 13),
            "ws": _host(ws, 17)}


@pytest.mark.parametrize("kind,status,msg", [("alloc", 6, b"workspace"),
                                             ("launch", 5, b"kernel launch"),
                                             ("sync", 5, b"synchronisation")])
def test_armed_fault_fires_once_and_touches_nothing(lib, kind, status, msg):
    bufs = _buffers(lib)
    before = {k: v.copy() for k, v in bufs.items()}
    bb.inject_fault(kind)
    assert _fit_call(lib, bufs) == status
    assert b"injected fault" in lib.aaac_last_error() and msg in lib.aaac_last_error()
    for k in bufs:
        assert np.array_equal(bufs[k], before[k]), k
    # disarmed: the next call gets past the hook (here it fails later, for
    # want of a device or because the buffers are host memory, but not with
    # the injected message)
    _fit_call(lib, bufs)
    assert b"injected fault" not in lib.aaac_last_error()


def test_argument_errors_come_before_the_fault(lib):
    """An invalid call still reports its own error (and keeps the fault armed
    for the next call that passes its checks)."""
    bufs = _buffers(lib)
    bb.inject_fault("launch")
    cfg = bb.Config(bb.INT4, 128, 16, 3).c()
    st = lib.aaac_fit_layer(_ptr(bufs["W"]), 64, 200, _ptr(bufs["I"]), _ptr(bufs["scales"]),
                            ctypes.byref(cfg), _ptr(bufs["T"]), None, None, _ptr(bufs["ws"]),
                            bufs["ws"].size, None)
    assert st == 2  # K not a multiple of g
    assert _fit_call(lib, bufs) == 5
    assert b"injected fault" in lib.aaac_last_error()
    bb.inject_fault(None)


def test_unknown_kind_is_rejected(lib):
    assert lib.aaac_inject_fault(b"disk") == 1
    bb.inject_fault(None)


def test_environment_variable_arms_one_fault():
    code = ("import ctypes, numpy as np\n"
            "from activation_aware_codebook_b200 import binding as bb\n"
            "from tests.test_fault_injection import _buffers, _fit_call\n"
            "lib = bb.load()\n"
            "b = _buffers(lib)\n"
            "print(_fit_call(lib, b), lib.aaac_last_error().decode())\n")
    env = dict(os.environ, AAAC_FAULT="alloc", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.startswith("6 injected fault: workspace"), out.stdout
