"""Oracle pins: AWQ-style pre-scaling before the fit.

"Technical summary: AAAC", section 4: AAAC combined with AWQ, which scales the
weights before quantisation, recovers more of the quantisation gap.  The page
gives no formula for the scaling; reading R16 takes the channel statistic from
the importance vector (v_k = I_k / tokens), c_k = v_k^(alpha/2) normalised by
sqrt(max * min), alpha = j/16, and a plain grid search over j that keeps the
first candidate with the lowest fitted objective.  Each pin below holds the
oracle to something other than its own code: identities of the definition,
closed forms, numpy's pow, the activations recomputed from X, and the plain
fit of the rescaled layer.
"""
import numpy as np
import pytest

import oracle
from activation_aware_codebook_b200 import synth


def _f32_of_bf16(h):
    return (np.asarray(h, dtype=np.uint32) << 16).view(np.float32)


def _layer(N, K, seed, T=64, heavy=True, dist="normal"):
    W, X = synth.small_layer(N, K, seed, T=T, heavy=heavy, dist=dist)
    return synth.bits_u16(W), synth.bits_u16(X)


def test_alpha_zero_is_the_identity():
    Wb, Xb = _layer(24, 256, 1)
    I = oracle.importance(Xb)
    c, Is, Ws = oracle.awq_prescale(Wb, I, Xb.shape[0], 0)
    assert np.all(c == 1.0)
    assert np.array_equal(Is.view(np.uint32), I.view(np.uint32))
    assert np.array_equal(Ws, Wb)


@pytest.mark.parametrize("j", range(17))
def test_equal_importance_gives_unit_scales(j):
    I = np.full(64, 3.7, dtype=np.float32)
    Wb, _ = _layer(4, 64, 2)
    c, Is, Ws = oracle.awq_prescale(Wb, I, 1000, j)
    assert np.all(c == 1.0)
    assert np.array_equal(Is, I) and np.array_equal(Ws, Wb)


@pytest.mark.parametrize("j", range(17))
def test_two_level_importance_closed_form(j):
    """Channel energies in ratio 2^16: p_hi / p_lo = 2^(j/2), so the
    normalised scales are exactly 2^(+j/4) and 2^(-j/4) (fp32-rounded when
    j/4 is not an integer)."""
    tokens = 77
    I = np.array([tokens, tokens * 65536.0] * 8, dtype=np.float32)
    Wb, _ = _layer(2, 16, 3)
    c, Is, _ = oracle.awq_prescale(Wb, I, tokens, j)
    assert np.all(c[0::2] == np.float32(2.0 ** (-j / 4)))
    assert np.all(c[1::2] == np.float32(2.0 ** (j / 4)))
    if j % 4 == 0:  # powers of two: I' exact
        assert np.all(Is[0::2] == np.float32(tokens * 2.0 ** (j / 2)))
        assert np.all(Is[1::2] == np.float32(tokens * 65536.0 * 2.0 ** (-j / 2)))


@pytest.mark.parametrize("j", [1, 3, 5, 8, 11, 16])
def test_scales_match_numpy_pow(j):
    rng = np.random.default_rng(5 + j)
    K, tokens = 4096, 2048
    I = (np.exp(rng.normal(0, 3, K)) * tokens).astype(np.float32)
    I[::97] = 0.0  # dead channels
    Wb, _ = _layer(2, K, 4)
    c, Is, _ = oracle.awq_prescale(Wb, I, tokens, j)
    live = I > 0
    p = np.power(I[live].astype(np.float64) / tokens, j / 32.0)
    ref = (p / np.sqrt(p.max() * p.min())).astype(np.float32)
    got = c[live]
    ulp = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1
    assert np.mean(ulp == 0) > 0.999
    assert np.all(c[~live] == 1.0) and np.all(Is[~live] == 0.0)


def test_dead_channels_do_not_move_the_normalisation():
    rng = np.random.default_rng(9)
    K = 512
    I = (np.exp(rng.normal(0, 2, K)) * 100).astype(np.float32)
    Wb, _ = _layer(2, K, 6)
    c_all, _, _ = oracle.awq_prescale(Wb, I, 100, 12)
    I2 = I.copy()
    I2[::5] = 0.0
    c_dead, Is_dead, _ = oracle.awq_prescale(Wb, I2, 100, 12)
    live = I2 > 0
    # the normalisation is over live channels only: recompute it on them
    p = np.power(I[live].astype(np.float64) / 100, 12 / 32.0)
    ref = (p / np.sqrt(p.max() * p.min())).astype(np.float32)
    d = np.abs(c_dead[live].view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert d.max() <= 1
    assert np.all(c_dead[~live] == 1.0) and np.all(Is_dead[~live] == 0.0)
    assert not np.array_equal(c_all, c_dead)


@pytest.mark.parametrize("j", [4, 9, 16])
def test_rescaled_activations_have_the_scaled_importance(j):
    """I' is the energy of x / c, recomputed here from X itself."""
    Wb, Xb = _layer(8, 384, 7, T=96)
    I = oracle.importance(Xb)
    c, Is, _ = oracle.awq_prescale(Wb, I, Xb.shape[0], j)
    x = _f32_of_bf16(Xb).astype(np.float64)
    e = ((x / c.astype(np.float64)[None, :]) ** 2).sum(axis=0)
    np.testing.assert_allclose(Is.astype(np.float64), e, rtol=2.0 ** -22, atol=0)
    assert c.max() / c.min() > 4  # heavy channels: the scales really vary


@pytest.mark.parametrize("j", [4, 9, 16])
def test_scaled_layer_computes_the_same_map(j):
    """(x / c) W'^T = x W^T up to the bf16 rounding of W' (relative 2^-8 per
    weight, plus the fp32 rounding of w * c)."""
    Wb, Xb = _layer(16, 256, 8)
    I = oracle.importance(Xb)
    c, _, Ws = oracle.awq_prescale(Wb, I, Xb.shape[0], j)
    w = _f32_of_bf16(Wb).astype(np.float64)
    ws = _f32_of_bf16(Ws).astype(np.float64) / c.astype(np.float64)[None, :]
    assert np.all(np.abs(ws - w) <= np.abs(w) * (2.0 ** -8 + 2.0 ** -22))
    # and W' really is scaled by c (not by 1/c): the big-c columns grew
    big = c > 2
    assert big.any()
    assert np.all(np.abs(_f32_of_bf16(Ws)[:, big]) >= np.abs(_f32_of_bf16(Wb)[:, big]))


@pytest.mark.parametrize("fmt,g,S", [(oracle.INT4, 128, 16), (oracle.NVFP4, 16, 16)])
def test_search_candidates_are_plain_fits_of_the_rescaled_layer(fmt, g, S):
    N, K, iters = 24, 256, 3
    Wb, Xb = _layer(N, K, 10 + S, dist="student_t4" if fmt == oracle.NVFP4 else "normal")
    I = oracle.importance(Xb)
    js = [0, 4, 8, 12, 16]
    res = oracle.awq_search(Wb, I, Xb.shape[0], fmt, g, S, iters, js)
    # alpha = 0 is the plain fit of the original layer
    plain = oracle.run_layer(Wb, Xb, fmt, g, S, iters)
    assert res["err_alpha"][0] == plain["err_final"]
    for idx, j in enumerate(js):
        c, Is, Ws = oracle.awq_prescale(Wb, I, Xb.shape[0], j)
        scl, T0 = oracle.init_codebooks(Ws, fmt, g)
        T, _, _ = oracle.fit(Ws, Is, scl, T0, fmt, g, S, iters)
        out = oracle.pack(Ws, Is, scl, T, fmt, g, S)
        assert res["err_alpha"][idx] == out["err_final"]
        if idx == res["best"]:
            assert np.array_equal(res["codes"], out["codes"])
            assert np.array_equal(res["c"], c)
    e = res["err_alpha"]
    assert res["best"] == int(np.argmin(e)) and e[res["best"]] == e.min()


def test_search_is_never_worse_than_the_plain_fit():
    """alpha = 0 is a candidate, so the kept objective is at most the plain
    fit's.  On these synthetic layers (independent weights, no structure
    linking large weights to large activations) the scaling often does not
    help the activation-weighted objective, and the search then keeps
    alpha = 0; the page's gain from combining with AWQ is measured on real
    models, which are not available here."""
    Wb, Xb = _layer(64, 512, 12, T=128)
    I = oracle.importance(Xb)
    res = oracle.awq_search(Wb, I, Xb.shape[0], oracle.INT4, 128, 16, 4, [0, 4, 8, 12, 16])
    plain = oracle.run_layer(Wb, Xb, oracle.INT4, 128, 16, 4)
    assert res["err_final"] <= plain["err_final"]
    assert res["err_alpha"][0] == plain["err_final"]
