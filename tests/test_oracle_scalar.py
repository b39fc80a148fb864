"""Oracle pins: number formats, scales and the normalised weights u.

Scales follow "Technical summary: AAAC" section 1 (the 4-bit format fixes the
code count and the per-group scale; g=128 INT4, g=16 NVFP4) read as R1:
INT4 s = bf16_RN(fp32_RN(absmax / 7)), NVFP4 s = e4m3_RN_satfinite(absmax).
They are pinned here by torch's own bf16 and float8_e4m3fn conversions, which
are library routines independent of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import synth


def _torch_bf16_bits(x_f32):
    t = torch.from_numpy(np.asarray(x_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_rn_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(4000).astype(np.float32) * np.float32(3.0)
    bits = x.view(np.uint32)
    # exact ties: low 16 bits 0x8000 with both parities of the kept LSB
    ties = ((bits[:500] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    edge = np.array([0.0, -0.0, 1e-40, -1e-40, 3.3e38, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9],
                    dtype=np.float32)
    for arr in (x, ties, edge):
        assert np.array_equal(oracle.f32_to_bf16_rn(arr), _torch_bf16_bits(arr))


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f32(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.all(np.isnan(ours[~finite]))
    assert oracle.e4m3_to_f32(np.array([0x7E]))[0] == 448.0


def test_e4m3_encode_matches_torch_in_range_and_saturates():
    rng = np.random.default_rng(2)
    a = np.abs(rng.standard_normal(5000)).astype(np.float32) * np.float32(0.05)
    a = np.concatenate([a, np.abs(rng.standard_normal(2000)).astype(np.float32) * 60,
                        np.array([0, 2 ** -10, 2 ** -9, 3 * 2 ** -11, 2 ** -6, 447.9, 416, 440],
                                 dtype=np.float32)])
    # every midpoint between consecutive finite codes (ties go to even)
    vals = oracle.e4m3_to_f32(np.arange(0, 0x7F, dtype=np.uint8)).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    a = np.concatenate([a, mids])
    a = a[a < 448]
    ours = oracle.f32_to_e4m3_rn_sat(a)
    ref = torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    big = np.array([448.0, 449.0, 463.9, 464.0, 1e6, np.inf], dtype=np.float32)
    assert np.all(oracle.f32_to_e4m3_rn_sat(big) == 0x7E)


@pytest.mark.parametrize("fmt,g", [(oracle.INT4, 128), (oracle.INT4, 32), (oracle.NVFP4, 16)])
def test_scales_closed_form(fmt, g):
    W = synth.make_weight(48, 256, seed=11)
    Wb = synth.bits_u16(W)
    got = oracle.scales(Wb, fmt, g)
    a = W.float().abs().reshape(48, 256 // g, g).amax(-1)
    if fmt == oracle.INT4:
        ref = (a / 7.0).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    else:
        ref = a.clamp(max=448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_scales_zero_group_and_tiny():
    W = torch.zeros(2, 32, dtype=torch.bfloat16)
    W[1, 16:] = 1e-4  # NVFP4: e4m3 of 1e-4 underflows to 0
    got = oracle.scales(synth.bits_u16(W), oracle.NVFP4, 16)
    assert got.tolist() == [[0, 0], [0, 0]]
    got = oracle.scales(synth.bits_u16(W), oracle.INT4, 16)
    assert got[0].tolist() == [0, 0] and got[1, 0] == 0 and got[1, 1] != 0


@pytest.mark.parametrize("fmt,g", [(oracle.INT4, 128), (oracle.NVFP4, 16)])
def test_u_is_w_times_fp32_reciprocal(fmt, g):
    W = synth.make_weight(16, 256, seed=5)
    Wb = synth.bits_u16(W)
    scl = oracle.scales(Wb, fmt, g)
    s = oracle.decode_scales(scl, fmt)
    u = oracle.u_values(Wb, scl, fmt, g)
    w = oracle.bf16_to_f32(Wb)
    with np.errstate(divide="ignore"):
        r = np.where(s > 0, np.float32(1) / s, np.float32(0)).astype(np.float32)
    ref = (w.reshape(16, -1, g) * r[:, :, None]).astype(np.float32).reshape(16, 256)
    assert np.array_equal(u.view(np.uint32), ref.view(np.uint32))
