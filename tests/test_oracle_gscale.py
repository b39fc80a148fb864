"""Oracle pins: NVFP4 with a per-tensor fp32 scale (reading R17).

"Technical summary: AAAC", section 1 and section 4 (the NVFP4 g=16 layout: a
4-bit code and an E4M3 scale per 16 weights) and section 2, core mechanism 3
(the choice in the sign bit of the positive scale).  The page does not say
whether NVFP4's per-tensor fp32 scale is used; reading R17 adds it as a
separate format: gs = fp32_RN(amax / 448), s8 = e4m3_RN_satfinite(fp32_RN(a /
gs)), effective scale fp32_RN(gs * s8).  The pins hold the oracle to torch's
own E4M3 conversion, to the plain NVFP4 path (a power-of-two tensor scale
with every group scale in E4M3's normal range reduces to it exactly), to
exact power-of-two scale invariance, to the E4M3 rounding bound, and to a
hand-worked dequantisation.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import synth


def _bf16(x):
    return synth.bits_u16(torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


def _f32(h):
    return (np.asarray(h, dtype=np.uint32) << 16).view(np.float32)


def _layer(N, K, seed, sigma, T=64):
    W, X = synth.small_layer(N, K, seed, T=T, heavy=True)
    w = W.float().numpy() * np.float32(sigma / 0.02)
    return _bf16(w), synth.bits_u16(X)


def test_scales_match_torch_e4m3():
    Wb, _ = _layer(32, 256, 1, 0.02)
    w = _f32(Wb)
    gs = oracle.global_scale(Wb)
    assert gs == np.float32(np.abs(w).max()) / np.float32(448.0)
    a = np.abs(w).reshape(32, 16, 16).max(axis=2).astype(np.float32)
    ref = torch.from_numpy(a / np.float32(gs)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.scales(Wb, oracle.NVFP4_GS, 16, gs)
    assert np.array_equal(got, ref)
    assert got.max() == 0x7E  # the largest group sits at 448


def test_power_of_two_tensor_scale_reduces_to_plain_nvfp4():
    """amax = 1.75 gives gs = 2^-8 exactly; with every group absmax inside
    E4M3's normal range both before and after the shift, s8 = 2^8 s and the
    effective scales, u, tables, codes and objectives all coincide."""
    N, K = 40, 256
    Wb, Xb = _layer(N, K, 2, 0.3)
    w = np.clip(_f32(Wb), -1.7, 1.7)
    w[0, 0] = 1.75
    Wb = _bf16(w)
    a = np.abs(_f32(Wb)).reshape(N, -1, 16).max(axis=2)
    assert a.min() >= 2.0 ** -6
    plain = oracle.run_layer(Wb, Xb, oracle.NVFP4, 16, 16, 4)
    gsr = oracle.run_layer(Wb, Xb, oracle.NVFP4_GS, 16, 16, 4)
    assert gsr["gs"] == 2.0 ** -8
    s_plain = oracle.decode_scales(plain["scales"], oracle.NVFP4)
    s8 = oracle.decode_scales(gsr["scales"], oracle.NVFP4_GS)
    assert np.array_equal(s8, s_plain * 256)
    assert np.array_equal(oracle.u_values(Wb, gsr["scales"], oracle.NVFP4_GS, 16, gsr["gs"]),
                          oracle.u_values(Wb, plain["scales"], oracle.NVFP4, 16))
    for k in ("T_init", "T", "T_bf16", "codes", "err_hist"):
        assert np.array_equal(gsr[k], plain[k]), k
    assert gsr["err_final"] == plain["err_final"]


def test_exact_power_of_two_invariance():
    """W * 2^-12: the tensor scale takes the factor, s8 and u do not change,
    and both objectives scale by 2^-24 exactly."""
    N, K = 32, 256
    Wb, Xb = _layer(N, K, 3, 0.02)
    W2 = _bf16(_f32(Wb) * np.float32(2.0 ** -12))
    assert np.array_equal(_f32(W2), _f32(Wb) * np.float32(2.0 ** -12))
    r1 = oracle.run_layer(Wb, Xb, oracle.NVFP4_GS, 16, 16, 4)
    r2 = oracle.run_layer(W2, Xb, oracle.NVFP4_GS, 16, 16, 4)
    assert r2["gs"] == r1["gs"] * 2.0 ** -12
    for k in ("scales", "T_init", "T", "T_bf16", "codes", "scales_tagged"):
        assert np.array_equal(r1[k], r2[k]), k
    assert np.array_equal(r2["err_hist"], r1["err_hist"] * 2.0 ** -24)
    assert r2["err_final"] == r1["err_final"] * 2.0 ** -24


def test_small_weights_keep_normal_scales():
    """Group maxima of about 2e-3 are E4M3 subnormals (quantum 2^-9) in plain
    NVFP4; with the tensor scale every effective scale is within E4M3's
    relative rounding bound 2^-4 of its group maximum, and the fit is better."""
    N, K = 48, 256
    Wb, Xb = _layer(N, K, 4, 1e-3)
    a = np.abs(_f32(Wb)).reshape(N, -1, 16).max(axis=2).astype(np.float64)
    gs = oracle.global_scale(Wb)
    s8 = oracle.decode_scales(oracle.scales(Wb, oracle.NVFP4_GS, 16, gs), oracle.NVFP4_GS)
    s_eff = (np.float32(gs) * s8.astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(s_eff - a) <= a * (2.0 ** -4 + 2.0 ** -20))
    s_plain = oracle.decode_scales(oracle.scales(Wb, oracle.NVFP4, 16), oracle.NVFP4)
    assert np.any(np.abs(s_plain - a) > a * 2.0 ** -4)
    plain = oracle.run_layer(Wb, Xb, oracle.NVFP4, 16, 16, 4)
    gsr = oracle.run_layer(Wb, Xb, oracle.NVFP4_GS, 16, 16, 4)
    assert gsr["err_final"] < plain["err_final"]


@pytest.mark.parametrize("S", [16, 8])
def test_round_trip_with_tensor_scale(S):
    N, K = 24, 320
    Wb, Xb = _layer(N, K, 5, 0.02)
    out = oracle.run_layer(Wb, Xb, oracle.NVFP4_GS, 16, S, 3)
    w_hat, ch = oracle.unpack(out["codes"], out["scales_tagged"], out["choice_bits"],
                              out["T_bf16"], N, K, oracle.NVFP4_GS, 16, S, out["gs"])
    w = _f32(Wb).astype(np.float64)
    err = (out["I"][None, :].astype(np.float64) * (w - w_hat) ** 2).sum()
    assert np.isclose(err, out["err_final"], rtol=1e-12, atol=0)
    # w_hat is the exact product of the effective scale and the table value
    s8 = oracle.decode_scales(out["scales_tagged"], oracle.NVFP4_GS)
    s_eff = (np.float32(out["gs"]) * s8).astype(np.float64)
    tv = _f32(out["T_bf16"]).astype(np.float64)
    q = np.concatenate([out["codes"][:, :, None] & 15, out["codes"][:, :, None] >> 4],
                       axis=2).reshape(N, K)
    c = np.repeat(ch, S, axis=1)
    assert np.array_equal(w_hat, np.repeat(s_eff, 16, axis=1) * tv[c, q])


def test_zero_tensor_is_all_dead():
    N, K = 4, 64
    Wb = np.zeros((N, K), dtype=np.uint16)
    Xb, = [synth.bits_u16(synth.make_activations(16, K, 6, True))]
    out = oracle.run_layer(Wb, Xb, oracle.NVFP4_GS, 16, 16, 2)
    assert out["gs"] == 0.0
    assert np.all(out["scales"] == 0)
    assert out["stats"].dead_groups == N * K // 16
    assert out["err_final"] == 0.0


def test_dequant_hand_worked():
    """One row of 16 weights, S = g = 16, s8 = 2.0 (E4M3 0x40), gs = fp32(0.1):
    s_eff = fp32(0.2); w_hat = bf16_RN(fp32_RN(s_eff * T0[q])), each value
    worked out with numpy fp32 arithmetic and torch's bf16 rounding."""
    T = np.zeros((2, 16), dtype=np.float32)
    T[0, :15] = np.linspace(-1.0, 1.0, 15).astype(np.float32)
    T[1, :15] = np.linspace(-0.9, 1.1, 15).astype(np.float32)
    Tb = _bf16(T)
    q = np.arange(16) % 15
    codes = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)[None, :]
    gs = float(np.float32(0.1))
    for tagged_byte, book in ((0x40, 0), (0xC0, 1)):
        tagged = np.array([[tagged_byte]], dtype=np.uint8)
        got = oracle.dequant_bf16(codes, tagged, None, Tb, 1, 16, oracle.NVFP4_GS, 16, 16, gs)
        s_eff = np.float32(np.float32(0.1) * np.float32(2.0))
        prod = (s_eff * _f32(Tb)[book, q]).astype(np.float32)
        ref = synth.bits_u16(torch.from_numpy(prod).to(torch.bfloat16))[None, :]
        assert np.array_equal(got, ref)
