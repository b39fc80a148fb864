"""Oracle pins: nearest-entry assignment, group error, codebook choice, and
the exact fixed-point terms of the refine sums.

"Technical summary: AAAC", section 2, core mechanism 4 (assign: each weight to
its entry; refine: Voronoi cells) and core mechanism 2 (each group takes the
codebook with the lower activation-weighted error).  Readings R4 (nearest by
exact distance, lowest index on a tie) and R5 (fp64 sequential error, T0 wins
a tie) are pinned by brute-force exact rational enumeration.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._exact import argmin_nearest, frac_f32


def _check(T, us):
    T = np.asarray(T, dtype=np.float32)
    us = np.asarray(us, dtype=np.float32)
    q = oracle.assign(T, len(T), us)
    ref = [argmin_nearest(T, u) for u in us]
    assert q.tolist() == ref, (T, us, q, ref)
    return q


def test_assign_random_matches_bruteforce():
    rng = np.random.default_rng(7)
    for trial in range(20):
        n = 16 if trial % 2 else 15
        T = np.sort(rng.standard_normal(n).astype(np.float32) * 3)
        u = rng.standard_normal(300).astype(np.float32) * 4
        _check(T, u)


def test_assign_midpoints_and_ties():
    assert _check([0.0, 1.0], [0.5, np.nextafter(np.float32(0.5), np.float32(1))]).tolist() == [0, 1]
    # midpoint 1 + 2^-24 is not an fp32 value
    a = np.float32(1.0)
    b = np.nextafter(a, np.float32(2))
    assert _check([a, b], [a, b]).tolist() == [0, 1]
    # duplicates: the lower duplicate always wins, the upper one is never used
    assert _check([0.0, 1.0, 1.0, 2.0], [1.2, 1.7, 1.0, 0.9]).tolist() == [1, 3, 1, 1]
    # signed zeros are equal values
    assert _check([-0.0, 0.0, 1.0], [0.0, -0.0, 1e-30, 0.4]).tolist() == [0, 0, 0, 0]


def test_assign_extreme_exponent_gap():
    # exact distances differ below fp64 resolution of 0.25
    assert _check([-(2.0 ** -60), 0.5], [0.25]).tolist() == [1]
    assert _check([2.0 ** -60, 0.5], [0.25]).tolist() == [0]
    assert _check([-(2.0 ** -100), 2.0 ** 20], [2.0 ** 19]).tolist() == [1]


def test_group_error_is_sequential_fp64_and_close_to_exact():
    rng = np.random.default_rng(8)
    for S in (8, 16, 128):
        u = rng.standard_normal(S).astype(np.float32) * 3
        I = np.abs(rng.standard_normal(S)).astype(np.float32) * 100
        T = np.sort(rng.standard_normal(16).astype(np.float32) * 3)
        q = oracle.assign(T, 16, u)
        D = oracle.group_error(u, I, T, q)
        seq = 0.0
        for i in range(S):
            e = float(u[i]) - float(T[q[i]])
            seq = seq + float(I[i]) * (e * e)
        assert D == seq
        exact = sum(frac_f32(I[i]) * (frac_f32(u[i]) - frac_f32(T[q[i]])) ** 2 for i in range(S))
        assert abs(Fraction(D) - exact) <= exact * Fraction(1, 10 ** 13)


def test_choice_and_codes_bruteforce_on_tiny_layer():
    """Both codebooks enumerated per group with exact rationals; the packed
    codes and choice bits must equal the brute-force argmin / argmin."""
    from activation_aware_codebook_b200 import synth
    N, K, g, S = 6, 64, 32, 16
    W = synth.make_weight(N, K, seed=21)
    X = synth.make_activations(16, K, seed=22, heavy=True)
    Wb, Xb = synth.bits_u16(W), synth.bits_u16(X)
    I = oracle.importance(Xb)
    scl = oracle.scales(Wb, oracle.INT4, g)
    u = oracle.u_values(Wb, scl, oracle.INT4, g)
    rng = np.random.default_rng(23)
    T = np.zeros((2, 16), dtype=np.float32)
    for c in range(2):  # bf16-exact tables, so packing does not move them
        T[c] = oracle.bf16_to_f32(oracle.f32_to_bf16_rn(np.sort(rng.uniform(-7, 7, 16))))
    out = oracle.pack(Wb, I, scl, T, oracle.INT4, g, S)
    w_hat, ch = oracle.unpack(out["codes"], out["scales_tagged"], out["choice_bits"],
                              out["T_bf16"], N, K, oracle.INT4, g, S)
    codes = np.zeros((N, K), dtype=np.int64)
    codes[:, 0::2] = out["codes"] & 15
    codes[:, 1::2] = out["codes"] >> 4
    s = oracle.decode_scales(scl, oracle.INT4)
    n_checked = 0
    for r in range(N):
        for j in range(K // S):
            ks = range(j * S, (j + 1) * S)
            q = [[argmin_nearest(T[c], u[r, k]) for k in ks] for c in range(2)]
            D = [sum(frac_f32(I[k]) * (frac_f32(u[r, k]) - frac_f32(T[c][qq])) ** 2
                     for k, qq in zip(ks, q[c])) for c in range(2)]
            if abs(D[1] - D[0]) <= max(D) * Fraction(1, 10 ** 12):
                continue  # a tie at fp64 resolution: fp64 rounding decides
            c = 1 if D[1] < D[0] else 0
            assert ch[r, j] == c
            assert codes[r, list(ks)].tolist() == q[c]
            n_checked += 1
    assert n_checked >= N * (K // S) - 1
    assert ch.sum() > 0 and ch.sum() < ch.size  # both books used


def test_round_mul_exact():
    """Refine terms: floor of the exact product in even columns, ceil in odd."""
    rng = np.random.default_rng(9)
    for _ in range(2000):
        I = np.float32(abs(rng.standard_normal()) * 10.0 ** rng.integers(-3, 4))
        s = np.float32(abs(rng.standard_normal()))
        a = float(np.ldexp(np.float64(I) * np.float64(s) * np.float64(s), int(rng.integers(0, 30))))
        u = np.float32(rng.standard_normal() * 4)
        x = Fraction(a) * frac_f32(u)
        assert oracle.round_mul(a, u, False) == math.floor(x)
        assert oracle.round_mul(a, u, True) == math.ceil(x)
    # halves, exact integers, products below one, signs, zero
    cases = [(2.5, 1.0), (-2.5, 1.0), (1.25, -2.0), (1.25, 6.0), (3.0, 2.0), (-3.0, 2.0),
             (2.0 ** -40, 1.5), (2.0 ** -40, -1.5), (0.0, 3.0), (5.0, 0.0), (2.0 ** 50, 1.0)]
    for a, u in cases:
        x = Fraction(a) * Fraction(u)
        assert oracle.round_mul(a, np.float32(u), False) == math.floor(x), (a, u)
        assert oracle.round_mul(a, np.float32(u), True) == math.ceil(x), (a, u)
    assert oracle.round_mul(2.5, np.float32(1.0), False) == 2
    assert oracle.round_mul(-2.5, np.float32(1.0), False) == -3
    assert oracle.round_mul(-2.5, np.float32(1.0), True) == -2


@pytest.mark.parametrize("M", [1, 1000, 2 ** 20, 58720256, 141557760])
def test_fixed_point_bound(M):
    rng = np.random.default_rng(M % 1000)
    I_max = float(np.float32(abs(rng.standard_normal()) * 1e6))
    S2_max = float(np.float32(0.04) ** 2)
    U_max = 7.03
    L = oracle.fixed_point_L(M, I_max, S2_max, U_max)
    B = min(40, 61 - int(np.ceil(np.log2(M))) if M > 1 else 61)
    B = min(B, 40)
    top = Fraction(I_max) * Fraction(S2_max) * Fraction(U_max) * Fraction(2) ** L
    assert top < Fraction(2) ** B <= Fraction(2) ** 40
    assert top >= Fraction(2) ** (B - 4)  # tight to within the three exponents
    assert M * Fraction(2) ** B <= Fraction(2) ** 61
