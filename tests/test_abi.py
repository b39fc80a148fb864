"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/aaac.h declares, sizes its workspace, and rejects
invalid arguments before launching anything."""
import ctypes
import os
import re

import pytest

from activation_aware_codebook_b200 import binding
from activation_aware_codebook_b200.csrc import build as cbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "aaac.h")


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return binding.load()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(aaac_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert "aaac_fit_layer" in syms and len(syms) >= 7
    for s in syms:
        assert hasattr(lib, s), s
    assert set(binding.EXPORTS) <= set(syms)
    assert b"sm_100a" in lib.aaac_version()


def test_struct_layouts_match_header():
    assert ctypes.sizeof(binding.CConfig) == 32
    assert ctypes.sizeof(binding.CStats) == 48


def test_workspace_size_monotone(lib):
    cfg = binding.Config(binding.INT4, 128, 16, 20)
    small = binding.workspace_size(cfg, 256, 512, 128)
    big = binding.workspace_size(cfg, 14336, 4096, 262144)
    assert 256 <= small < big
    # the fit keeps an fp32 (s, 1/s) pair per scale group, the pack one choice
    # byte per selection group (S < g): the workspace holds either
    assert binding.workspace_size(cfg, 4096, 4096) >= 4096 * (4096 // 128) * 8
    assert binding.workspace_size(cfg, 4096, 4096) >= 4096 * (4096 // 16)
    nv = binding.Config(binding.NVFP4, 16, 16, 20)
    assert binding.workspace_size(nv, 4096, 4096) >= 4096 * (4096 // 16) * 8
    assert lib.aaac_workspace_size(None, 0, 0, 0) == 256


def _cfg(**kw):
    return binding.Config(**kw).c()


@pytest.mark.parametrize("kw,status", [
    (dict(fmt=3), 4), (dict(fmt=2, g=16, S=16), 1), (dict(fmt=2, g=32), 4), (dict(fmt=1, g=32), 4), (dict(g=48), 4), (dict(S=4), 2), (dict(S=256), 2),
    (dict(S=24), 2), (dict(iters=-1), 1), (dict(flags=16), 1)])
def test_invalid_config_rejected_without_launch(lib, kw, status):
    c = _cfg(**kw)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    st = lib.aaac_init_codebooks(fake, 64, 256, ctypes.byref(c), fake, fake, fake, 1 << 30, None)
    assert st == status, lib.aaac_last_error()
    assert lib.aaac_last_error()


def test_invalid_shapes_and_pointers(lib):
    c = _cfg()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lib.aaac_fit_layer(fake, 64, 200, fake, fake, ctypes.byref(c), fake, None, None, fake,
                              1 << 30, None) == 2  # K % g
    assert lib.aaac_fit_layer(fake, 1 << 20, 4096, fake, fake, ctypes.byref(c), fake, None, None,
                              fake, 1 << 30, None) == 2  # N*K >= 2^31
    assert lib.aaac_fit_layer(None, 64, 256, fake, fake, ctypes.byref(c), fake, None, None, fake,
                              1 << 30, None) == 1
    assert lib.aaac_fit_layer(odd, 64, 256, fake, fake, ctypes.byref(c), fake, None, None, fake,
                              1 << 30, None) == 3
    assert lib.aaac_fit_layer(fake, 64, 256, fake, fake, ctypes.byref(c), fake, None, None, fake,
                              16, None) == 6
    assert lib.aaac_fit_layer(fake, 64, 256, fake, fake, ctypes.byref(c), fake, None, None, None,
                              1 << 30, None) == 6
    assert lib.aaac_fit_layer(fake, 64, 256, fake, fake, None, fake, None, None, fake, 1 << 30,
                              None) == 1
    # S < g needs choice_bits
    c16 = _cfg(S=16)
    assert lib.aaac_pack(fake, 64, 256, fake, fake, ctypes.byref(c16), fake, fake, fake, fake,
                         None, None, fake, 1 << 30, None) == 1
    # importance
    assert lib.aaac_importance(fake, 0, 256, 256, 0, fake, fake, 1 << 30, None) == 2
    assert lib.aaac_importance(fake, 16, 250, 256, 0, fake, fake, 1 << 30, None) == 3
    assert lib.aaac_importance(fake, 16, 256, 128, 0, fake, fake, 1 << 30, None) == 2
    assert lib.aaac_importance(fake, 16, 256, 256, 4, fake, fake, 1 << 30, None) == 1
    assert lib.aaac_importance(fake, 16, 256, 256, 0, fake, fake, 8, None) == 6


def test_binding_refuses_without_cuda(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(RuntimeError):
        binding.importance(torch.zeros(8, 8, dtype=torch.bfloat16))


def test_awq_entry_points_validate_before_anything(lib):
    """Every call below has NULL device pointers, so no path can reach a
    launch; the status shows which check refused it."""
    assert lib.aaac_awq_prescale(None, 4, 60, None, 10, 3, None, None, None, None) == 3  # K % 8
    assert lib.aaac_awq_prescale(None, 4, 64, None, 0, 3, None, None, None, None) == 2   # tokens
    assert lib.aaac_awq_prescale(None, 4, 64, None, 10, 17, None, None, None, None) == 1  # alpha
    assert lib.aaac_awq_prescale(None, 4, 64, None, 10, 3, None, None, None, None) == 1   # W NULL
    c = _cfg()
    js = (ctypes.c_int32 * 2)(0, 20)
    assert lib.aaac_awq_fit(None, 64, 256, None, 10, ctypes.byref(c), js, 2, None, None, None,
                            None, None, None, None, None, None, 0, None) == 1  # alpha16[1]
    assert lib.aaac_awq_fit(None, 64, 256, None, 10, ctypes.byref(c), None, 1, None, None, None,
                            None, None, None, None, None, None, 0, None) == 1  # alpha16 NULL
    assert lib.aaac_awq_fit(None, 64, 200, None, 10, ctypes.byref(c), js, 1, None, None, None,
                            None, None, None, None, None, None, 0, None) == 2  # K % g


def test_awq_workspace_size(lib):
    c = _cfg()
    small = lib.aaac_awq_workspace_size(ctypes.byref(c), 64, 256)
    big = lib.aaac_awq_workspace_size(ctypes.byref(c), 128, 512)
    assert 0 < small < big
    # at least the rescaled weights, the codes and the fit's own workspace
    assert small >= 64 * 256 * 2 + 64 * 128 + lib.aaac_workspace_size(ctypes.byref(c), 64, 256, 0)
    assert lib.aaac_awq_workspace_size(ctypes.byref(c), 64, 200) == 0
    assert lib.aaac_awq_workspace_size(None, 64, 256) == 0
