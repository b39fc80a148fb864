"""Oracle pin for the near-tie count of the choice.

"Technical summary: AAAC", section 2, core mechanism 2: each selection group
takes the codebook with the lower activation-weighted error.  The parity
contract counts the groups whose two errors differ by less than 1e-6 of the
larger one (reading R13); those are the only groups whose choice may depend on
rounding, so the count must itself be right.

The layer is built by hand so that both errors are known exactly:
  * one row, INT4 with g = S = 16, so every group has its own scale and its
    own importance values;
  * each group holds w = 7 (its absmax, so s = 7/7 = 1 and u = w exactly), one
    w = 1/2, and zeros whose importance is 0;
  * T0 = {-8, ..., 7} and T1 = T0 + 1/2 (both exact in bf16).
The weight 7 sits on T0 and halfway between 6.5 and 7.5 (the lower wins), the
weight 1/2 sits on T1 and halfway between 0 and 1; so D0 = I_b / 4 and
D1 = I_a / 4 for the importance I_a of the 7 and I_b of the 1/2.  With I_a and
I_b one and one-plus-a-few-ulps, |D1 - D0| / max = 8 ulps (9.54e-7, a near
tie) or 9 ulps (1.07e-6, not one) of 1.
"""
import numpy as np

import oracle

ULP1 = 2.0 ** -23  # fp32 spacing just above 1
BF16_7 = 0x40E0    # 7.0
BF16_HALF = 0x3F00  # 0.5

# (I of the 7, I of the 1/2, near tie?, expected choice)
GROUPS = [
    (1.0, 1.0, True, 0),                                   # equal errors: tie, T0
    (1.0 + 8 * ULP1, 1.0, True, 0),                         # D1 above D0 by 9.54e-7
    (1.0 + 9 * ULP1, 1.0, False, 0),                        # D1 above D0 by 1.07e-6
    (1.0, 1.0 + 8 * ULP1, True, 1),                         # D0 above D1: near, T1 wins
    (1.0, 1.0 + 9 * ULP1, False, 1),                        # D0 above D1: not near
    ((1.0 + 8 * ULP1) * 2.0 ** 20, 2.0 ** 20, True, 0),     # relative, not absolute
    ((1.0 + 9 * ULP1) * 2.0 ** -20, 2.0 ** -20, False, 0),
]


def _layer():
    K = 16 * len(GROUPS)
    W = np.zeros((1, K), dtype=np.uint16)
    I = np.zeros(K, dtype=np.float32)
    for j, (ia, ib, _, _) in enumerate(GROUPS):
        W[0, 16 * j] = BF16_7
        W[0, 16 * j + 1] = BF16_HALF
        I[16 * j] = np.float32(ia)
        I[16 * j + 1] = np.float32(ib)
    assert all(np.float32(ia) == ia and np.float32(ib) == ib for ia, ib, _, _ in GROUPS)
    T = np.zeros((2, 16), dtype=np.float32)
    T[0] = np.arange(-8, 8, dtype=np.float32)
    T[1] = T[0] + 0.5
    return W, I, T


def test_hand_built_groups_have_unit_scales_and_exact_u():
    W, I, T = _layer()
    scl, _ = oracle.init_codebooks(W, oracle.INT4, 16)
    assert np.all(oracle.decode_scales(scl, oracle.INT4) == 1.0)
    u = oracle.u_values(W, scl, oracle.INT4, 16)
    assert np.all(u[0, ::16] == 7.0) and np.all(u[0, 1::16] == 0.5)


def test_near_tie_count_of_the_pack_assign():
    W, I, T = _layer()
    scl, _ = oracle.init_codebooks(W, oracle.INT4, 16)
    out = oracle.pack(W, I, scl, T, oracle.INT4, 16, 16)
    assert out["near_ties"] == sum(1 for g in GROUPS if g[2])
    _, choice = oracle.unpack(out["codes"], out["scales_tagged"], out["choice_bits"],
                              out["T_bf16"], 1, W.shape[1], oracle.INT4, 16, 16)
    assert [int(c) for c in choice[0]] == [g[3] for g in GROUPS]


def test_near_tie_count_of_a_fit_round_with_frozen_books():
    """The fit counts the ties of its last round's assign: with both books
    frozen that assign sees exactly T, so the count is the pack's."""
    W, I, T = _layer()
    scl, _ = oracle.init_codebooks(W, oracle.INT4, 16)
    flags = oracle.FREEZE_T0 | oracle.FREEZE_T1
    T_out, err, st = oracle.fit(W, I, scl, T, oracle.INT4, 16, 16, 2, flags)
    assert np.array_equal(T_out, T)
    assert st.near_ties == sum(1 for g in GROUPS if g[2])
    assert st.groups_t1 == sum(g[3] for g in GROUPS)
    # the objective of the round is the sum of the chosen errors (s = 1)
    want = sum((ia if c else ib) / 4.0 for ia, ib, _, c in GROUPS)
    assert np.allclose(err, want, rtol=1e-15)


def test_single_codebook_still_counts_near_ties():
    """The count is about the two errors, not about which book is used."""
    W, I, T = _layer()
    scl, _ = oracle.init_codebooks(W, oracle.INT4, 16)
    flags = oracle.FREEZE_T0 | oracle.FREEZE_T1 | oracle.SINGLE_CODEBOOK
    _, _, st = oracle.fit(W, I, scl, T, oracle.INT4, 16, 16, 1, flags)
    assert st.near_ties == sum(1 for g in GROUPS if g[2])
    assert st.groups_t1 == 0
