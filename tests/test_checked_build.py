"""The debugging build with device-side index checks (build.py --checks).

On the CPU: the normal library reports that it is not a checked build and its
check flag reads 0 without touching a device.  On the GPU: the checked library
runs whole layers of both formats and several group sizes in a
child process, gives the same tables as the normal library, and every check
holds (flag 0).
"""
import ctypes
import os
import subprocess
import sys

import pytest

from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200.csrc import build as cbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_normal_build_reports_no_checks():
    cbuild.build()
    lib = bb.load()
    assert lib.aaac_checked_build() == 0
    v = ctypes.c_uint32(7)
    assert lib.aaac_device_checks(ctypes.byref(v)) == 0
    assert v.value == 0
    assert lib.aaac_device_checks(None) == 1  # AAAC_ERR_INVALID_ARG


_CHILD = r"""
import sys, torch
from activation_aware_codebook_b200 import binding as bb, synth
assert bb.load().aaac_checked_build() == 1, "not the checked build"
dev = torch.device("cuda", 0)
out = []
for (N, K, fmt, g, S, it, seed) in [(256, 512, bb.INT4, 128, 16, 6, 1),
                                     (384, 1024, bb.NVFP4, 16, 16, 6, 2),
                                     (200, 2048, bb.NVFP4, 16, 8, 4, 3),
                                     (130, 768, bb.INT4, 128, 128, 5, 4)]:
    W = synth.make_weight(N, K, seed, "normal" if seed % 2 else "student_t4", device=dev)
    X = synth.make_activations(512, K, seed + 100, bool(seed % 2), device=dev)
    r = bb.run_layer(W, X, bb.Config(fmt, g, S, it))
    torch.cuda.synchronize()
    out.append(r["T"].view(torch.int32).cpu())
torch.save(out, sys.argv[1])
print("CHECKS", bb.device_checks())
"""


@pytest.mark.gpu
def test_checked_build_runs_clean_and_agrees(tmp_path):
    cbuild.build(checks=True)
    env = dict(os.environ, AAAC_CHECKED="1", PYTHONPATH=ROOT)
    res = subprocess.run([sys.executable, "-c", _CHILD, str(tmp_path / "checked.pt")], env=env,
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    assert "CHECKS 0" in res.stdout, res.stdout
    env["AAAC_CHECKED"] = "0"
    res2 = subprocess.run([sys.executable, "-c", _CHILD.replace(
        'assert bb.load().aaac_checked_build() == 1, "not the checked build"', ""),
        str(tmp_path / "plain.pt")], env=env, cwd=ROOT, capture_output=True, text=True,
        timeout=600)
    assert res2.returncode == 0, res2.stderr[-3000:]
    import torch
    a = torch.load(tmp_path / "checked.pt")
    b = torch.load(tmp_path / "plain.pt")
    assert all(torch.equal(x, y) for x, y in zip(a, b))
