"""Oracle pins: column importance I_k = sum_t X[t,k]^2.

"Technical summary: AAAC", section 2, core mechanism 2 defines I_k as the
activation energy of input column k over the calibration set.  Reading R0:
I_k = fp32_RN(exact sum).  The pin is a brute-force exact rational sum rounded
to fp32 by tests/_exact.py, plus cases built so that a plain fp64 running sum
lands on the wrong side of an fp32 rounding boundary.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from activation_aware_codebook_b200 import synth
from tests._exact import f32_rn


def _bf16(vals):
    return synth.bits_u16(torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16))


def _exact_I(Xb, init=None):
    T, K = Xb.shape
    x = oracle.bf16_to_f32(Xb)
    out = []
    for k in range(K):
        s = Fraction(0) if init is None else Fraction(float(init[k]))
        for t in range(T):
            v = Fraction(float(x[t, k]))
            s += v * v
        out.append(f32_rn(s))
    return np.array(out, dtype=np.float32)


def test_importance_random_equals_exact_sum():
    X = synth.make_activations(96, 40, seed=3, heavy=True)
    Xb = synth.bits_u16(X)
    got = oracle.importance(Xb)
    assert np.array_equal(got.view(np.uint32), _exact_I(Xb).view(np.uint32))
    # and it is the sum of squares to fp64 accuracy
    ref = (oracle.bf16_to_f32(Xb).astype(np.float64) ** 2).sum(0)
    assert np.allclose(got, ref, rtol=1e-7, atol=0)


def test_importance_rounding_boundary_cases():
    # 2^24 + 1 is the exact midpoint of fp32 2^24 and 2^24+2: ties to even give
    # 2^24, but a tiny extra term must push it up.  A plain fp64 running sum
    # drops the tiny term and rounds down.
    col0 = [4096.0, 1.0, 2.0 ** -60, 0.0]
    col1 = [4096.0, 1.0, 0.0, 0.0]           # exact tie -> even (2^24)
    col2 = [4096.0, 1.0, -(2.0 ** -60), 2.0 ** -61]
    col3 = [1e-39, -1e-39, 2.0 ** -130, 0.0]  # bf16 subnormals -> 0 in fp32
    col4 = [2.0 ** 64, 0.0, 0.0, 0.0]         # 2^128 overflows fp32
    cols = [col0, col1, col2, col3, col4]
    Xb = np.stack([_bf16(c) for c in cols], axis=1)
    got = oracle.importance(Xb)
    assert got[0] == np.float32(2.0 ** 24 + 2)
    assert got[1] == np.float32(2.0 ** 24)
    assert got[2] == np.float32(2.0 ** 24 + 2)
    assert got[3] == 0.0
    assert np.isinf(got[4])
    assert np.array_equal(got.view(np.uint32), _exact_I(Xb).view(np.uint32))
    naive = (oracle.bf16_to_f32(Xb).astype(np.float64) ** 2).sum(0).astype(np.float32)
    assert naive[0] != got[0]  # the case really separates exact from fp64


def test_importance_accumulate_and_stride():
    X = synth.make_activations(50, 24, seed=9, heavy=False)
    Xb = synth.bits_u16(X)
    I1 = oracle.importance(Xb[:20])
    I2 = oracle.importance(Xb[20:], I_in=I1)
    assert np.array_equal(I2.view(np.uint32), _exact_I(Xb[20:], init=I1).view(np.uint32))
    # a strided view of a wider buffer gives the same as the packed copy
    wide = np.zeros((50, 32), dtype=np.uint16)
    wide[:, :24] = Xb
    out = np.empty(24, dtype=np.float32)
    lib = oracle.lib()
    lib.orc_importance(wide.ctypes.data, 50, 24, 32, None, out.ctypes.data)
    assert np.array_equal(out, oracle.importance(Xb))


def test_exact_sumsq_single_terms():
    rng = np.random.default_rng(4)
    for v in rng.standard_normal(200).astype(np.float32) * 10:
        b = _bf16([float(v)])
        x = float(oracle.bf16_to_f32(b)[0])
        assert oracle.exact_sumsq_bf16(b) == np.float32(f32_rn(Fraction(x) ** 2))
