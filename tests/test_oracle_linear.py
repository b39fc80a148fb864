"""Oracle pins: inference dequantisation of the packed format and the W4A16
linear that consumes it.

"Technical summary: AAAC", section 1 (the dequantised values decide the
weights used at inference; W4A16) and section 2, core mechanism 3 (BF16 tables,
the group's choice in the sign bit of its positive scale, or in a bitmask when
S < g).  Reading R15: w_hat = bf16_RN(s * T_c[code]).
"""
import numpy as np
import torch

import oracle
from activation_aware_codebook_b200 import synth


def _bf16_bits(x):
    return synth.bits_u16(torch.tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16))


def _f32_of_bf16(h):
    return (np.asarray(h, dtype=np.uint32) << 16).view(np.float32)


def _codes(q):
    q = np.asarray(q, dtype=np.uint8)
    return (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)


def test_dequant_hand_built_int4_sign_bit():
    """Two rows, INT4 g = S = 16.  Row 0: scale 0.5 on T0 = {-8..7}.  Row 1:
    scale 0.75 with the sign bit set (T1 = 1 + q/128) and codes reversed.
    0.75 (1 + q/128) = (192 + 1.5 q)/256: even q is exact, odd q is a tie on
    the 1/256 grid of [0.5, 1) and rounds to the even numerator."""
    T = np.zeros((2, 16), dtype=np.uint16)
    T[0] = _bf16_bits(np.arange(16) - 8.0)
    T[1] = _bf16_bits(1.0 + np.arange(16) / 128.0)
    q = np.zeros((2, 16), dtype=np.uint8)
    q[0] = np.arange(16)
    q[1] = 15 - np.arange(16)
    scales = np.array([[0x3F00], [0x3F40 | 0x8000]], dtype=np.uint16)  # 0.5; -0.75 = choice 1
    w = oracle.dequant_bf16(_codes(q), scales, None, T, 2, 16, oracle.INT4, 16, 16)
    num1 = {0: 192, 1: 194, 2: 195, 3: 196, 4: 198, 5: 200, 6: 201, 7: 202,
            8: 204, 9: 206, 10: 207, 11: 208, 12: 210, 13: 212, 14: 213, 15: 214}
    expect0 = (np.arange(16) - 8.0) / 2
    expect1 = np.array([num1[15 - k] / 256.0 for k in range(16)])
    assert np.array_equal(_f32_of_bf16(w[0]), expect0.astype(np.float32))
    assert np.array_equal(_f32_of_bf16(w[1]), expect1.astype(np.float32))


def test_dequant_hand_built_bitmask_and_nvfp4():
    # INT4 g=32, S=16: the choice of group j is bit j of the row's bitmask
    T = np.zeros((2, 16), dtype=np.uint16)
    T[0] = _bf16_bits(np.arange(16) * 0.25)
    T[1] = _bf16_bits(-np.arange(16) * 1.0)
    q = np.full((1, 32), 3, dtype=np.uint8)
    scales = np.array([[0x3F80]], dtype=np.uint16)  # 1.0, sign bit clear when S < g
    bits = np.array([[0b10]], dtype=np.uint8)       # group 0 -> T0, group 1 -> T1
    w = _f32_of_bf16(oracle.dequant_bf16(_codes(q), scales, bits, T, 1, 32, oracle.INT4, 32, 16))
    assert np.all(w[0, :16] == 0.75) and np.all(w[0, 16:] == -3.0)
    # NVFP4 g = S = 16: E4M3 0x40 = 2.0, tagged 0xC0 -> T1 = q/2
    T[1] = _bf16_bits(np.arange(16) * 0.5)
    q = np.arange(16, dtype=np.uint8)[None, :] % 15
    w = _f32_of_bf16(oracle.dequant_bf16(_codes(q), np.array([[0xC0]], dtype=np.uint8), None, T,
                                         1, 16, oracle.NVFP4, 16, 16))
    assert np.array_equal(w[0], (np.arange(16) % 15).astype(np.float32))


def test_dequant_rtn_matches_textbook_int4():
    """Books frozen to the uniform grid {-8..7}: the packed layer dequantises
    to bf16_RN(s * (q - 8)), computed here with numpy and torch."""
    N, K, g = 16, 256, 128
    W = synth.make_weight(N, K, 5)
    Wb = synth.bits_u16(W)
    Xb = synth.bits_u16(synth.make_activations(64, K, 6, False))
    I = oracle.importance(Xb)
    scl, _ = oracle.init_codebooks(Wb, oracle.INT4, g)
    grid = np.zeros((2, 16), dtype=np.float32)
    grid[0] = grid[1] = np.arange(16) - 8.0
    out = oracle.pack(Wb, I, scl, grid, oracle.INT4, g, g,
                      oracle.FREEZE_T0 | oracle.FREEZE_T1)
    w = oracle.dequant_bf16(out["codes"], out["scales_tagged"], out.get("choice_bits"),
                            out["T_bf16"], N, K, oracle.INT4, g, g)
    codes = out["codes"]
    q = np.empty((N, K), dtype=np.int64)
    q[:, 0::2] = codes & 15
    q[:, 1::2] = codes >> 4
    s = _f32_of_bf16(np.asarray(out["scales_tagged"], dtype=np.uint16) & 0x7FFF).astype(np.float64)
    ref = _bf16_bits(np.repeat(s, g, axis=1) * (q - 8.0))
    assert np.array_equal(w, ref)


def test_linear_one_hot_and_matmul():
    rng = np.random.default_rng(3)
    N, K = 12, 96
    Wh = _bf16_bits(rng.standard_normal((N, K)))
    # one-hot rows of X pick single columns of w_hat exactly
    X = np.zeros((4, K), dtype=np.float64)
    cols = [0, 5, 47, 95]
    for i, c in enumerate(cols):
        X[i, c] = 1.0
    Y = oracle.linear(_bf16_bits(X), Wh)
    for i, c in enumerate(cols):
        assert np.array_equal(Y[i], _f32_of_bf16(Wh[:, c]).astype(np.float64))
    # random X against numpy's fp64 matmul of the same bf16 values
    Xb = _bf16_bits(rng.standard_normal((5, K)))
    Y = oracle.linear(Xb, Wh)
    ref = _f32_of_bf16(Xb).astype(np.float64) @ _f32_of_bf16(Wh).astype(np.float64).T
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)
