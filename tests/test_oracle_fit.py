"""Oracle pins for the fit and the pack.

"Technical summary: AAAC", section 2, core mechanism 4: quantile
initialisation (T1 offset by half a step), then alternating assign and
weighted-centroid refine; section 2, core mechanism 3 and section 4: BF16
tables, choice in the scale's sign bit, S=16 at 0.0625 bpw.

Pins (none re-types the oracle's own formula):
  * init = numpy.sort order statistics at the evenly spaced ranks;
  * fixed uniform INT4 grid -> round-to-nearest (the RTN baseline the page
    compares against), with half-way cases going down;
  * equal importance, one codebook, equal scales -> plain 1-D Lloyd k-means
    written here in numpy;
  * one refine = the I*s^2-weighted mean of each cell (closed form);
  * the objective never increases; codebooks stay sorted and inside the data;
  * the printed storage figures and a round trip through the packed format.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from activation_aware_codebook_b200 import synth
from tests._exact import total_order_keys

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "storage_arithmetic.txt")


def _layer(N, K, seed, T=32, heavy=True, dist="normal"):
    W, X = synth.small_layer(N, K, seed, T=T, heavy=heavy, dist=dist)
    return synth.bits_u16(W), synth.bits_u16(X)


@pytest.mark.parametrize("fmt,g", [(oracle.INT4, 128), (oracle.NVFP4, 16)])
def test_init_is_sorted_order_statistics(fmt, g):
    Wb, _ = _layer(40, 256, seed=31)
    scl, T = oracle.init_codebooks(Wb, fmt, g)
    u = oracle.u_values(Wb, scl, fmt, g).ravel()
    keys = np.sort(total_order_keys(u))
    srt = u[np.argsort(total_order_keys(u), kind="stable")]
    M = u.size
    n = oracle.ncodes(fmt)
    for j in range(n):
        r0 = ((2 * j + 1) * M) // (2 * n)
        r1 = min(M - 1, ((j + 1) * M) // n)
        assert T[0, j].view(np.uint32) == srt[r0].view(np.uint32)
        assert T[1, j].view(np.uint32) == srt[r1].view(np.uint32)
    assert np.all(T[:, n:] == 0)
    assert np.all(np.diff(keys.astype(np.int64)) >= 0)
    # T1 sits half a step above T0: T0_j <= T1_j <= T0_{j+1}
    assert np.all(T[0, :n] <= T[1, :n]) and np.all(T[1, :n - 1] <= T[0, 1:n])


def test_rtn_special_case():
    """Both books frozen to the uniform INT4 grid {-8..7}: codes are
    round-to-nearest of u (ties down), every group on T0, T unchanged."""
    N, K, g = 24, 512, 128
    Wb, Xb = _layer(N, K, seed=41)
    I = oracle.importance(Xb)
    scl = oracle.scales(Wb, oracle.INT4, g)
    grid = np.arange(-8, 8, dtype=np.float32)
    T = np.stack([grid, grid])
    flags = oracle.FREEZE_T0 | oracle.FREEZE_T1
    Tf, err, st = oracle.fit(Wb, I, scl, T, oracle.INT4, g, g, 3, flags)
    assert np.array_equal(Tf, T)
    assert st.groups_t1 == 0
    out = oracle.pack(Wb, I, scl, Tf, oracle.INT4, g, g, flags)
    u = oracle.u_values(Wb, scl, oracle.INT4, g).astype(np.float64)
    rtn = np.clip(np.ceil(u - 0.5), -8, 7).astype(np.int64)  # half-way -> down
    codes = np.zeros((N, K), dtype=np.int64)
    codes[:, 0::2] = out["codes"] & 15
    codes[:, 1::2] = out["codes"] >> 4
    assert np.array_equal(codes - 8, rtn)
    assert np.all((out["scales_tagged"] >> 15) == 0)
    # informational: disagreement with torch.round (half-to-even) only at ties
    half_even = np.clip(np.round(u), -8, 7)
    differ = half_even != rtn
    assert np.all((u - np.floor(u))[differ] == 0.5)
    # objective: sum over groups s^2 * sum I (u - q)^2 with q = rtn
    s = oracle.decode_scales(scl, oracle.INT4).astype(np.float64)
    D = (I[None, :].astype(np.float64) * (u - rtn) ** 2).reshape(N, K // g, g).sum(-1)
    assert np.allclose(err, (s ** 2 * D).sum(), rtol=1e-12)


def _lloyd_numpy(u, T, iters):
    """Textbook 1-D Lloyd k-means on u (equal weights)."""
    T = np.array(T, dtype=np.float32)
    for _ in range(iters):
        Ts = np.sort(T.astype(np.float64))
        mids = (Ts[:-1] + Ts[1:]) / 2
        idx = np.searchsorted(mids, u.astype(np.float64), side="left")  # u on a midpoint -> lower
        for j in range(len(Ts)):
            m = idx == j
            if m.any():
                Ts[j] = np.float32(u[m].astype(np.float64).mean())
        T = np.sort(Ts.astype(np.float32))
    return T


def test_kmeans_special_case():
    """I == 1, a single codebook and one +-A weight per group (so all scales
    are equal): the fit is plain 1-D k-means on u."""
    N, K, g = 32, 256, 128
    rng = np.random.default_rng(51)
    w = rng.uniform(-0.019, 0.019, (N, K)).astype(np.float32)
    A = np.float32(0.02)
    w[:, ::g] = A * np.where(rng.random((N, K // g)) < 0.5, 1, -1)
    Wb = synth.bits_u16(torch.from_numpy(w).to(torch.bfloat16))
    Xb = synth.bits_u16(torch.ones(1, K, dtype=torch.bfloat16))
    I = oracle.importance(Xb)
    assert np.all(I == 1.0)
    scl, T0 = oracle.init_codebooks(Wb, oracle.INT4, g)
    assert len(np.unique(scl)) == 1
    u = oracle.u_values(Wb, scl, oracle.INT4, g).ravel()
    T1, _, _ = oracle.fit(Wb, I, scl, T0, oracle.INT4, g, g, 1, oracle.SINGLE_CODEBOOK)
    ref1 = _lloyd_numpy(u, T0[0], 1)
    diff = np.abs(T1[0].view(np.int32).astype(np.int64) - ref1.view(np.int32).astype(np.int64))
    assert diff.max() <= 1 and (diff == 0).mean() >= 0.9
    assert np.array_equal(T1[1], T0[1])  # the unused book never moves
    Tn, err, _ = oracle.fit(Wb, I, scl, T0, oracle.INT4, g, g, 60, oracle.SINGLE_CODEBOOK)
    refn = _lloyd_numpy(u, T0[0], 60)
    assert np.allclose(Tn[0], refn, rtol=1e-6, atol=1e-6)


def test_one_refine_is_weighted_mean():
    N, K, g, S = 32, 256, 128, 16
    Wb, Xb = _layer(N, K, seed=61)
    I = oracle.importance(Xb).astype(np.float64)
    scl, T0 = oracle.init_codebooks(Wb, oracle.INT4, g)
    u = oracle.u_values(Wb, scl, oracle.INT4, g).astype(np.float64)
    s = oracle.decode_scales(scl, oracle.INT4).astype(np.float64)
    A = I[None, :] * np.repeat(s ** 2, g, axis=1)
    # the assignment the first iteration uses, from numpy
    q = np.stack([np.searchsorted((T0[c, :-1].astype(np.float64) + T0[c, 1:]) / 2, u,
                                  side="left") for c in range(2)])
    err = np.stack([(I[None, :] * (u - T0[c][q[c]]) ** 2).reshape(N, K // S, S).sum(-1)
                    for c in range(2)])
    choice = (err[1] < err[0]).astype(np.int64)
    chw = np.repeat(choice, S, axis=1)
    T1, hist, _ = oracle.fit(Wb, oracle.importance(Xb), scl, T0, oracle.INT4, g, S, 1)
    ref = T0.astype(np.float64).copy()
    for c in range(2):
        for j in range(16):
            m = (chw == c) & (q[c] == j)
            if m.any():
                ref[c, j] = (A[m] * u[m]).sum() / A[m].sum()
        ref[c] = np.sort(ref[c])
    assert np.allclose(T1.astype(np.float64), ref, rtol=2e-7, atol=0)
    # it minimises the cell objective: moving any entry by +-eps does not help
    for c in range(2):
        for j in range(16):
            m = (chw == c) & (q[c] == j)
            if not m.any():
                continue
            t = float(T1[c][np.argmin(np.abs(T1[c] - ref[c, j]))])
            f = lambda x: (A[m] * (u[m] - x) ** 2).sum()
            eps = 1e-3 * max(abs(t), 1e-3)
            assert f(t) <= f(t + eps) and f(t) <= f(t - eps)
    assert hist[0] > 0


@pytest.mark.parametrize("fmt,g,S,dist", [(oracle.INT4, 128, 128, "normal"),
                                          (oracle.INT4, 128, 16, "normal"),
                                          (oracle.NVFP4, 16, 16, "student_t4"),
                                          (oracle.NVFP4, 16, 8, "student_t4")])
def test_objective_monotone_and_books_sorted(fmt, g, S, dist):
    N, K = 48, 512
    Wb, Xb = _layer(N, K, seed=71 + S, dist=dist)
    I = oracle.importance(Xb)
    scl, T = oracle.init_codebooks(Wb, fmt, g)
    u = oracle.u_values(Wb, scl, fmt, g)
    n = oracle.ncodes(fmt)
    hist = []
    for it in range(8):
        T, err, st = oracle.fit(Wb, I, scl, T, fmt, g, S, 1)
        hist.append(err[0])
        for c in range(2):
            assert np.all(np.diff(T[c, :n]) >= 0)
            assert T[c, :n].min() >= u.min() and T[c, :n].max() <= u.max()
    hist = np.array(hist)
    assert np.all(hist[1:] <= hist[:-1] * (1 + 1e-9)), hist
    assert hist[-1] < hist[0]
    # a multi-iteration call is the same as repeated single calls
    _, T0 = oracle.init_codebooks(Wb, fmt, g)
    Tm, errm, _ = oracle.fit(Wb, I, scl, T0, fmt, g, S, 8)
    assert np.array_equal(Tm, T) and np.array_equal(errm, hist)


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


@pytest.mark.parametrize("fmt,g,S", [(oracle.INT4, 128, 128), (oracle.INT4, 128, 16),
                                     (oracle.NVFP4, 16, 16), (oracle.NVFP4, 16, 8)])
def test_pack_storage_arithmetic_and_round_trip(fmt, g, S):
    gold = _golden()
    N, K = 32, 512
    Wb, Xb = _layer(N, K, seed=81)
    out = oracle.run_layer(Wb, Xb, fmt, g, S, 4)
    assert out["T_bf16"].nbytes == gold["codebook_bytes_per_layer"]
    assert out["T_bf16"].size == gold["codebook_entries_per_layer"]
    assert gold["layers_7b"] * out["T_bf16"].nbytes == gold["codebook_bytes_7b"]
    assert round(gold["codebook_bytes_7b"] / 1024) == gold["codebook_kib_7b_approx"]
    assert out["codes"].nbytes * 2 == N * K  # 4 bits per weight
    if S == g:
        assert out["choice_bits"] is None
        assert out["scales_tagged"].nbytes == out["scales"].nbytes  # S = g: no extra bytes
        assert gold["extra_bytes_S_eq_g"] == 0
    else:
        extra_bpw = out["choice_bits"].nbytes * 8 / (N * K)
        assert extra_bpw == 1.0 / S
        if S == 16 and g == 128:
            assert extra_bpw == gold["extra_bpw_S16_g128"]
    n = oracle.ncodes(fmt)
    codes = np.concatenate([out["codes"] & 15, out["codes"] >> 4], axis=1)
    assert codes.max() < n
    w_hat, ch = oracle.unpack(out["codes"], out["scales_tagged"], out["choice_bits"],
                              out["T_bf16"], N, K, fmt, g, S)
    w = oracle.bf16_to_f32(Wb).astype(np.float64)
    err = (out["I"][None, :].astype(np.float64) * (w - w_hat.astype(np.float64)) ** 2).sum()
    assert np.isclose(err, out["err_final"], rtol=1e-12, atol=0)
    # tags sit in the sign bit only when S == g; magnitudes are untouched
    sign = 15 if fmt == oracle.INT4 else 7
    mask = (1 << sign) - 1
    assert np.array_equal(out["scales_tagged"] & mask, out["scales"])
    if S == g:
        assert np.array_equal((out["scales_tagged"] >> sign).astype(np.uint8), ch)
    else:
        assert np.all((out["scales_tagged"] >> sign) == 0)
    assert 0 < ch.sum() < ch.size
    # the packed fit is no worse than round-to-nearest on the uniform grid
    grid = (np.arange(-8, 8, dtype=np.float32) if fmt == oracle.INT4 else
            np.array([-6, -4, -3, -2, -1.5, -1, -0.5, 0, .5, 1, 1.5, 2, 3, 4, 6, 0],
                     dtype=np.float32) / 6)
    Tg = np.stack([grid, grid])
    rtn = oracle.pack(Wb, out["I"], out["scales"], Tg, fmt, g, S,
                      oracle.FREEZE_T0 | oracle.FREEZE_T1 | oracle.SINGLE_CODEBOOK)
    assert out["err_final"] < rtn["err_final"]
