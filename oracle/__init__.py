"""CPU oracle for the AAAC per-layer codebook fit -- TEST INFRASTRUCTURE.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline /
reference legs may import this package.  The product path (the CUDA library
``activation_aware_codebook_b200``) never imports, links or calls it, and the
two share no code.  The arithmetic lives in ``aaac_oracle.c`` (plain C, fp64
and exact integer arithmetic); this module only marshals numpy arrays.

What each entry point follows ("Technical summary: AAAC", gist.science/ko/
paper/2605.08692) and what pins it (tests/test_oracle_*.py):

  importance        section 2 mech. 2 (I_k = sum_t X^2).  Pinned by an exact
                    rational sum rounded to fp32 in Python (fractions), on
                    random and hand-made boundary cases.
  scales            section 1 / 4 (g=128 INT4, g=16 NVFP4 group scales).
                    Pinned by torch's own bf16 / float8_e4m3fn conversions.
  u                 section 2 mech. 4 (normalised weights).  Pinned by numpy
                    fp32 arithmetic.
  init_codebooks    section 2 mech. 4, initialisation (quantiles, T1 offset
                    by half a step).  Pinned by numpy.sort at the ranks.
  assign            section 2 mech. 4, assign (nearest entry).  Pinned by a
                    brute-force exact (fractions) argmin, midpoint ties,
                    duplicates, signed zeros.
  group_error       section 2 mech. 2 (lower activation-weighted error).
                    Pinned by exact rational errors and brute-force choice.
  round_mul         exact fixed-point terms of the refine sums (floor in even
                    columns, ceil in odd ones).  Pinned by exact rational
                    floor / ceil.
  fit               section 2 mech. 4 (alternating assign / refine).  Pinned
                    by: the RTN special case (fixed uniform INT4 grid), the
                    plain 1-D k-means special case (equal importance, one
                    codebook, equal scales), the weighted-mean closed form of
                    one refine, monotone objective, sorted codebooks.
  pack / unpack     section 2 mech. 3 and section 4 (BF16 tables, sign-bit
                    choice, S=16 at 0.0625 bpw).  Pinned by the printed
                    storage arithmetic (tests/golden/storage_arithmetic.txt)
                    and by a round trip that recomputes err_final.
  dequant_bf16      section 1 (dequantised values used at inference, W4A16)
                    and section 2 mech. 3.  Pinned by a hand-built packed
                    layer with its values worked out by hand, and by the RTN
                    special case against numpy's textbook INT4 dequantisation.
  linear            Y = X W_hat^T in fp64.  Pinned by one-hot rows of X
                    (Y is a column of W_hat exactly) and by numpy's matmul.
  awq_prescale      section 4 (AAAC combined with AWQ's weight scaling before
                    quantisation; reading R16 for the scaling itself).  Pinned
                    by: alpha = 0 is the identity, equal importance gives unit
                    scales, a two-level importance gives 2^(+-j/4) in closed
                    form, numpy's pow within one fp32 ulp, the importance of
                    the rescaled activations recomputed from X, and the
                    scaled layer computing the same map within bf16 rounding.
  awq_search        plain grid search over alpha = j/16, keeping the first
                    candidate with the lowest err_final.  Pinned by: alpha = 0
                    reproduces the plain fit, and each candidate equals the
                    plain fit of its rescaled layer.
  Final fitted values of a whole run: parity unpinned by the pages (they print
  no worked example); held only by the pins above.
"""
import ctypes
import os

import numpy as np

from . import build as _build

INT4 = 0
NVFP4 = 1
NVFP4_GS = 2  # NVFP4 with a per-tensor fp32 scale (reading R17)
FREEZE_T0 = 1
FREEZE_T1 = 2
SINGLE_CODEBOOK = 4

_lib = None


class Stats(ctypes.Structure):
    _fields_ = [("near_ties", ctypes.c_int64), ("groups_t1", ctypes.c_int64),
                ("empty_cells", ctypes.c_int64), ("dead_groups", ctypes.c_int64),
                ("L", ctypes.c_int32), ("pad", ctypes.c_int32)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f32_to_bf16_rn.restype = ctypes.c_uint16
        L.orc_f32_to_bf16_rn.argtypes = [ctypes.c_float]
        L.orc_e4m3_to_f32.restype = ctypes.c_float
        L.orc_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.orc_f32_to_e4m3_rn_sat.restype = ctypes.c_uint8
        L.orc_f32_to_e4m3_rn_sat.argtypes = [ctypes.c_float]
        L.orc_exact_sumsq_bf16.restype = ctypes.c_float
        L.orc_exact_sumsq_bf16.argtypes = [P, i64, i64, ctypes.c_float]
        L.orc_importance.restype = None
        L.orc_importance.argtypes = [P, i64, i64, i64, P, P]
        L.orc_scales.restype = None
        L.orc_scales.argtypes = [P, i64, i64, i32, i32, P, ctypes.c_float]
        L.orc_u.restype = None
        L.orc_u.argtypes = [P, i64, i64, i32, i32, P, P, ctypes.c_float]
        L.orc_rank_t0.restype = i64
        L.orc_rank_t0.argtypes = [i64, i32, i32]
        L.orc_rank_t1.restype = i64
        L.orc_rank_t1.argtypes = [i64, i32, i32]
        L.orc_init_codebooks.restype = i32
        L.orc_init_codebooks.argtypes = [P, i64, i64, i32, i32, P, P, P]
        L.orc_global_scale.restype = ctypes.c_float
        L.orc_global_scale.argtypes = [P, i64, i64]
        L.orc_assign.restype = None
        L.orc_assign.argtypes = [P, i32, P, i64, P]
        L.orc_group_error.restype = ctypes.c_double
        L.orc_group_error.argtypes = [P, P, P, P, i32]
        L.orc_round_mul.restype = i64
        L.orc_round_mul.argtypes = [ctypes.c_double, ctypes.c_float, i32]
        L.orc_fixed_point_L.restype = i32
        L.orc_fixed_point_L.argtypes = [i64, ctypes.c_double, ctypes.c_double, ctypes.c_double]
        L.orc_fit.restype = i32
        L.orc_fit.argtypes = [P, i64, i64, P, P, i32, i32, i32, i32, ctypes.c_uint, P, P, P,
                              ctypes.c_float]
        L.orc_pack.restype = i32
        L.orc_pack.argtypes = [P, i64, i64, P, P, i32, i32, i32, ctypes.c_uint, P, P, P, P, P,
                               P, P, ctypes.c_float]
        L.orc_dequant_bf16.restype = None
        L.orc_dequant_bf16.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, P, ctypes.c_float]
        L.orc_linear.restype = None
        L.orc_linear.argtypes = [P, i64, i64, P, i64, i64, P]
        L.orc_unpack.restype = None
        L.orc_unpack.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, P, P, ctypes.c_float]
        L.orc_awq_scales.restype = None
        L.orc_awq_scales.argtypes = [P, i64, i64, i32, P, P]
        L.orc_awq_scale_weights.restype = None
        L.orc_awq_scale_weights.argtypes = [P, i64, i64, P, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def ncodes(fmt):
    return 16 if fmt == INT4 else 15


def scale_dtype(fmt):
    return np.uint16 if fmt == INT4 else np.uint8


# --- scalar formats ---------------------------------------------------------

def bf16_to_f32(h):
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_rn(x):
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib().orc_f32_to_bf16_rn(float(v)) for v in x], dtype=np.uint16)


def f32_to_e4m3_rn_sat(x):
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib().orc_f32_to_e4m3_rn_sat(float(v)) for v in x], dtype=np.uint8)


def e4m3_to_f32(b):
    b = np.asarray(b, dtype=np.uint8).ravel()
    return np.array([lib().orc_e4m3_to_f32(int(v)) for v in b], dtype=np.float32)


def decode_scales(scales, fmt):
    """Decoded magnitudes (sign / tag bit ignored), fp32."""
    s = np.asarray(scales)
    if fmt == INT4:
        return bf16_to_f32(s.astype(np.uint16) & 0x7FFF)
    table = e4m3_to_f32(np.arange(256, dtype=np.uint8))
    return table[s.astype(np.uint8) & 0x7F]


# --- the path ---------------------------------------------------------------

def exact_sumsq_bf16(x_u16, init=0.0):
    x = _u16(x_u16)
    return lib().orc_exact_sumsq_bf16(_p(x), x.size, 1, float(init))


def importance(X_u16, I_in=None, ldx=None):
    X = _u16(X_u16)
    T, K = X.shape
    out = np.empty(K, dtype=np.float32)
    I_in = None if I_in is None else np.ascontiguousarray(I_in, dtype=np.float32)
    lib().orc_importance(_p(X), T, K, ldx if ldx is not None else K, _p(I_in), _p(out))
    return out


def global_scale(W_u16):
    """Tensor scale of reading R17: fp32_RN(max |w| / 448), 0 for a zero tensor."""
    W = _u16(W_u16)
    N, K = W.shape
    return float(np.float32(lib().orc_global_scale(_p(W), N, K)))


def scales(W_u16, fmt, g, gs=0.0):
    W = _u16(W_u16)
    N, K = W.shape
    out = np.empty((N, K // g), dtype=scale_dtype(fmt))
    lib().orc_scales(_p(W), N, K, fmt, g, _p(out), float(gs))
    return out


def u_values(W_u16, scl, fmt, g, gs=0.0):
    W = _u16(W_u16)
    N, K = W.shape
    scl = np.ascontiguousarray(scl, dtype=scale_dtype(fmt))
    out = np.empty((N, K), dtype=np.float32)
    lib().orc_u(_p(W), N, K, fmt, g, _p(scl), _p(out), float(gs))
    return out


def rank_t0(M, n, j):
    return lib().orc_rank_t0(M, n, j)


def rank_t1(M, n, j):
    return lib().orc_rank_t1(M, n, j)


def init_codebooks(W_u16, fmt, g, with_gs=False):
    """(scales, T), or (scales, T, gs) with with_gs (gs = 0 unless NVFP4_GS)."""
    W = _u16(W_u16)
    N, K = W.shape
    scl = np.empty((N, K // g), dtype=scale_dtype(fmt))
    T = np.zeros((2, 16), dtype=np.float32)
    gs = np.zeros(1, dtype=np.float32)
    rc = lib().orc_init_codebooks(_p(W), N, K, fmt, g, _p(scl), _p(T), _p(gs))
    assert rc == 0
    return (scl, T, float(gs[0])) if with_gs else (scl, T)


def assign(T, n, u):
    T = np.ascontiguousarray(T, dtype=np.float32)
    u = np.ascontiguousarray(u, dtype=np.float32)
    q = np.empty(u.shape, dtype=np.uint8)
    lib().orc_assign(_p(T), n, _p(u), u.size, _p(q))
    return q


def group_error(u, Ik, Tc, q):
    u = np.ascontiguousarray(u, dtype=np.float32)
    Ik = np.ascontiguousarray(Ik, dtype=np.float32)
    Tc = np.ascontiguousarray(Tc, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.uint8)
    return lib().orc_group_error(_p(u), _p(Ik), _p(Tc), _p(q), u.size)


def round_mul(a, u, up):
    """floor(a*u) (up=False) or ceil(a*u) (up=True) of the exact product."""
    return lib().orc_round_mul(float(a), float(u), 1 if up else 0)


def fixed_point_L(M, I_max, S2_max, U_max):
    return lib().orc_fixed_point_L(M, I_max, S2_max, U_max)


def fit(W_u16, I, scl, T_init, fmt, g, S, iters, flags=0, gs=0.0):
    W = _u16(W_u16)
    N, K = W.shape
    I = np.ascontiguousarray(I, dtype=np.float32)
    scl = np.ascontiguousarray(scl, dtype=scale_dtype(fmt))
    T = np.array(T_init, dtype=np.float32).reshape(2, 16).copy()
    err = np.zeros(max(iters, 1), dtype=np.float64)
    st = Stats()
    rc = lib().orc_fit(_p(W), N, K, _p(I), _p(scl), fmt, g, S, iters, flags, _p(T), _p(err),
                       ctypes.cast(ctypes.pointer(st), ctypes.c_void_p), float(gs))
    assert rc == 0
    return T, err[:iters], st


def pack(W_u16, I, scl, T, fmt, g, S, flags=0, gs=0.0):
    W = _u16(W_u16)
    N, K = W.shape
    I = np.ascontiguousarray(I, dtype=np.float32)
    scl = np.ascontiguousarray(scl, dtype=scale_dtype(fmt))
    T = np.ascontiguousarray(T, dtype=np.float32).reshape(2, 16)
    T_bf16 = np.zeros((2, 16), dtype=np.uint16)
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    tagged = np.zeros_like(scl)
    nb = (K // S + 7) // 8
    bits = np.zeros((N, nb), dtype=np.uint8) if S != g else None
    err = np.zeros(1, dtype=np.float64)
    ties = np.zeros(1, dtype=np.int64)
    rc = lib().orc_pack(_p(W), N, K, _p(I), _p(scl), fmt, g, S, flags, _p(T), _p(T_bf16),
                        _p(codes), _p(tagged), _p(bits), _p(err), _p(ties), float(gs))
    assert rc == 0
    return dict(T_bf16=T_bf16, codes=codes, scales_tagged=tagged, choice_bits=bits,
                err_final=float(err[0]), near_ties=int(ties[0]))


def unpack(codes, scales_tagged, choice_bits, T_bf16, N, K, fmt, g, S, gs=0.0):
    """Exact dequantised values s * T_bf16[c][code] (fp64) and the choices."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    tagged = np.ascontiguousarray(scales_tagged, dtype=scale_dtype(fmt))
    bits = None if choice_bits is None else np.ascontiguousarray(choice_bits, dtype=np.uint8)
    T_bf16 = np.ascontiguousarray(T_bf16, dtype=np.uint16)
    w_hat = np.empty((N, K), dtype=np.float64)
    ch = np.empty((N, K // S), dtype=np.uint8)
    lib().orc_unpack(_p(codes), _p(tagged), _p(bits), _p(T_bf16), N, K, fmt, g, S, _p(w_hat),
                     _p(ch), float(gs))
    return w_hat, ch


def dequant_bf16(codes, scales_tagged, choice_bits, T_bf16, N, K, fmt, g, S, gs=0.0):
    """bf16 bits of bf16_RN(s * T_bf16[c][code]) per weight, [N, K] uint16
    (with a tensor scale: bf16_RN(fp32_RN(fp32_RN(gs * s8) * T)))."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    tagged = np.ascontiguousarray(scales_tagged, dtype=scale_dtype(fmt))
    bits = None if choice_bits is None else np.ascontiguousarray(choice_bits, dtype=np.uint8)
    T_bf16 = np.ascontiguousarray(T_bf16, dtype=np.uint16)
    w_hat = np.empty((N, K), dtype=np.uint16)
    lib().orc_dequant_bf16(_p(codes), _p(tagged), _p(bits), _p(T_bf16), N, K, fmt, g, S,
                           _p(w_hat), float(gs))
    return w_hat


def linear(X_u16, w_hat_u16):
    """Y = X @ w_hat^T in fp64 (k order), X [M, K] and w_hat [N, K] bf16 bits."""
    X = np.ascontiguousarray(X_u16, dtype=np.uint16)
    Wh = np.ascontiguousarray(w_hat_u16, dtype=np.uint16)
    M, K = X.shape
    N = Wh.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    lib().orc_linear(_p(X), M, K, _p(Wh), N, K, _p(Y))
    return Y


def run_layer(W_u16, X_u16, fmt, g, S, iters, flags=0):
    """importance -> init -> fit -> pack, all on the CPU."""
    I = importance(X_u16)
    scl, T0, gs = init_codebooks(W_u16, fmt, g, with_gs=True)
    T, err, st = fit(W_u16, I, scl, T0, fmt, g, S, iters, flags, gs)
    out = pack(W_u16, I, scl, T, fmt, g, S, flags, gs)
    out.update(I=I, scales=scl, T_init=T0, T=T, err_hist=err, stats=st, gs=gs)
    return out


def awq_prescale(W_u16, I, tokens, j):
    """(c, I', W') of reading R16 for alpha = j/16: per-channel scales, the
    importance of the rescaled activations, and the rescaled bf16 weights."""
    W = _u16(W_u16)
    N, K = W.shape
    I = np.ascontiguousarray(I, dtype=np.float32)
    c = np.empty(K, dtype=np.float32)
    Is = np.empty(K, dtype=np.float32)
    lib().orc_awq_scales(_p(I), K, int(tokens), int(j), _p(c), _p(Is))
    Ws = np.empty_like(W)
    lib().orc_awq_scale_weights(_p(W), N, K, _p(c), _p(Ws))
    return c, Is, Ws


def awq_search(W_u16, I, tokens, fmt, g, S, iters, js, flags=0):
    """Grid search over alpha = j/16 (j in js, ascending): fit and pack each
    rescaled layer and keep the first candidate with the lowest err_final."""
    js = [int(j) for j in js]
    errs = []
    best = None
    for idx, j in enumerate(js):
        c, Is, Ws = awq_prescale(W_u16, I, tokens, j)
        scl, T0, gs = init_codebooks(Ws, fmt, g, with_gs=True)
        T, err, st = fit(Ws, Is, scl, T0, fmt, g, S, iters, flags, gs)
        out = pack(Ws, Is, scl, T, fmt, g, S, flags, gs)
        errs.append(out["err_final"])
        if best is None or out["err_final"] < errs[best[0]]:
            out.update(c=c, I=Is, W=Ws, scales=scl, T=T, err_hist=err, stats=st, gs=gs)
            best = (idx, out)
    return dict(best=best[0], err_alpha=np.array(errs, dtype=np.float64), **best[1])
