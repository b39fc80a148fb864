/*
 * aaac_oracle.c -- plain CPU oracle for the AAAC per-layer codebook fit.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * product path (the CUDA library under activation_aware_codebook_b200/) never
 * links, imports or calls it, and it shares no code with that path.
 *
 * What it computes follows "Technical summary: AAAC (activation-aware
 * adaptive codebooks)" (gist.science/ko/paper/2605.08692):
 *   section 2, core mechanism 1   two scalar codebooks T0/T1 per layer with the
 *                                 format's cardinality (16 INT4, 15 NVFP4);
 *   section 2, core mechanism 2   per-group choice of the codebook with the
 *                                 lower activation-weighted error, weights
 *                                 I_k = sum_t X[t,k]^2;
 *   section 2, core mechanism 3   choice stored in the sign bit of the
 *                                 positive scale;
 *   section 2, core mechanism 4   quantile initialisation (T1 shifted by half
 *                                 a step), then alternating assign / weighted
 *                                 centroid refine.
 * The page leaves every rounding, tie and reduction precision open.  The
 * readings taken here (R0..R9) are written next to the code that applies
 * them; each is stated once more in the repository's design notes.
 *
 * Style: plain loops, fp64 where floating point is asked for, exact integer
 * arithmetic (128-bit products, a small fixed-size big integer) where the
 * result has to be exact.  OpenMP only splits loops over independent rows or
 * columns; every cross-row sum is either an integer sum (order-free) or is
 * taken sequentially afterwards in row-major order.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -fPIC -shared (see build.py).
 *
 * Parity status of each entry point is listed in the header comment of
 * oracle/__init__.py next to the pins that hold it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef unsigned __int128 u128;
typedef __int128 i128;

#define ORC_INT4 0
#define ORC_NVFP4 1
#define ORC_NVFP4_GS 2   /* NVFP4 with a per-tensor fp32 scale (reading R17) */
#define ORC_FREEZE_T0 1u
#define ORC_FREEZE_T1 2u
#define ORC_SINGLE_CODEBOOK 4u

/* ------------------------------------------------------------------------ */
/* scalar formats                                                            */
/* ------------------------------------------------------------------------ */

static float f32_of(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t bits_of(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

float orc_bf16_to_f32(uint16_t h) { return f32_of((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
uint16_t orc_f32_to_bf16_rn(float f)
{
    uint32_t b = bits_of(f);
    if ((b & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((b >> 16) | 0x40u);
    uint32_t keep_lsb = (b >> 16) & 1u;
    b += 0x7fffu + keep_lsb;
    return (uint16_t)(b >> 16);
}

/* E4M3 ("fn" variant): bias 7, 3 mantissa bits, no infinities, S.1111.111 is
 * NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.  Subnormals are
 * m/8 * 2^-6.                                                               */
float orc_e4m3_to_f32(uint8_t v)
{
    int sign = v >> 7, e = (v >> 3) & 15, m = v & 7;
    double mag;
    if (e == 15 && m == 7) return f32_of(0x7fc00000u);
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(8.0 + m, e - 10);
    return (float)(sign ? -mag : mag);
}

/* Non-negative fp32 -> E4M3, round to nearest even, saturating to 448. */
uint8_t orc_f32_to_e4m3_rn_sat(float x)
{
    if (!(x >= 0.0f)) return 0; /* only used on absolute maxima */
    if (x >= 448.0f) return 0x7e; /* 448 = e 15, m 6 */
    double xd = x;
    if (xd < ldexp(1.0, -6)) {            /* subnormal quantum 2^-9 */
        double q = nearbyint(ldexp(xd, 9)); /* 0..8; 8 is the smallest normal */
        int qi = (int)q;
        if (qi == 8) return (uint8_t)(1 << 3);
        return (uint8_t)qi;
    }
    int e2;
    frexp(xd, &e2);          /* xd in [2^(e2-1), 2^e2) */
    int e = e2 - 1;          /* unbiased exponent */
    double q = nearbyint(ldexp(xd, 3 - e)); /* in [8, 16] */
    int qi = (int)q;
    if (qi == 16) { qi = 8; e += 1; }
    int ef = e + 7;
    if (ef > 15 || (ef == 15 && qi - 8 > 6)) return 0x7e; /* saturate */
    return (uint8_t)((ef << 3) | (qi - 8));
}

/* ------------------------------------------------------------------------ */
/* a small unsigned big integer: 10 x 64-bit limbs, little-endian            */
/* ------------------------------------------------------------------------ */

#define NLIMB 10
typedef struct { uint64_t w[NLIMB]; } big_t;

static void big_zero(big_t* a) { memset(a, 0, sizeof(*a)); }

/* a += m * 2^pos, m < 2^64, pos >= 0 and pos + 64 < 64 * NLIMB. */
static void big_add_shifted(big_t* a, uint64_t m, int pos)
{
    int limb = pos >> 6, off = pos & 63;
    u128 v = (u128)m << off; /* up to 128 bits */
    uint64_t part[3];
    part[0] = (uint64_t)v;
    part[1] = (uint64_t)(v >> 64);
    part[2] = 0;
    uint64_t carry = 0;
    for (int i = limb; i < NLIMB; i++) {
        uint64_t add = (i - limb < 3) ? part[i - limb] : 0;
        u128 s = (u128)a->w[i] + add + carry;
        a->w[i] = (uint64_t)s;
        carry = (uint64_t)(s >> 64);
        if (i - limb >= 2 && carry == 0) break;
    }
}

static int big_cmp(const big_t* a, const big_t* b)
{
    for (int i = NLIMB - 1; i >= 0; i--) {
        if (a->w[i] != b->w[i]) return a->w[i] < b->w[i] ? -1 : 1;
    }
    return 0;
}

/* a - b, requires a >= b */
static void big_sub(big_t* r, const big_t* a, const big_t* b)
{
    uint64_t borrow = 0;
    for (int i = 0; i < NLIMB; i++) {
        u128 s = (u128)a->w[i] - b->w[i] - borrow;
        r->w[i] = (uint64_t)s;
        borrow = (uint64_t)(s >> 64) ? 1 : 0;
    }
}

static void big_addto(big_t* r, const big_t* a, const big_t* b)
{
    uint64_t carry = 0;
    for (int i = 0; i < NLIMB; i++) {
        u128 s = (u128)a->w[i] + b->w[i] + carry;
        r->w[i] = (uint64_t)s;
        carry = (uint64_t)(s >> 64);
    }
}

static int big_bit(const big_t* a, int pos) { return (int)((a->w[pos >> 6] >> (pos & 63)) & 1u); }

static int big_top(const big_t* a)
{
    for (int i = NLIMB - 1; i >= 0; i--)
        if (a->w[i]) return i * 64 + 63 - __builtin_clzll(a->w[i]);
    return -1;
}

/* The value a * 2^-lsb_exp rounded to fp32, nearest, ties to even. */
static float big_to_f32_rn(const big_t* a, int lsb_exp)
{
    int h = big_top(a);
    if (h < 0) return 0.0f;
    /* fp32 keeps 24 bits down to the subnormal quantum 2^-149 */
    int sub_pos = lsb_exp - 149; /* bit position of 2^-149 */
    int lo = h - 23;
    if (lo < sub_pos) lo = sub_pos;
    /* callers use lsb_exp >= 149, so lo >= 0 */
    uint64_t mant = 0;
    for (int p = h; p >= lo; p--) mant = (mant << 1) | (uint64_t)big_bit(a, p);
    int round = 0, sticky = 0;
    if (lo - 1 >= 0) {
        round = big_bit(a, lo - 1);
        for (int p = lo - 2; p >= 0 && !sticky; p--) sticky |= big_bit(a, p);
    }
    if (round && (sticky || (mant & 1u))) mant++;
    double v = ldexp((double)mant, lo - lsb_exp);
    return (float)v; /* exact, or overflow to +inf */
}

/* Exact value of an fp32 number as (sign, magnitude * 2^-149). */
static int big_of_f32(big_t* a, float x)
{
    big_zero(a);
    uint32_t b = bits_of(x);
    int sign = (int)(b >> 31);
    int e = (int)((b >> 23) & 255u);
    uint32_t m = b & 0x7fffffu;
    if (e == 0) { big_add_shifted(a, m, 0); }
    else { big_add_shifted(a, (uint64_t)(m | 0x800000u), e - 1); }
    return sign;
}

/* ------------------------------------------------------------------------ */
/* R0: column importance (section 2, core mechanism 2: I_k = sum_t X^2)     */
/*     I_k = fp32_RN( [I_in,k +] sum_t x_{t,k}^2 ), the sum taken exactly.   */
/* ------------------------------------------------------------------------ */

/* Exact big-integer sum with LSB 2^-268 (the square of the smallest bf16
 * subnormal is 2^-266). */
static void add_sq_bf16(big_t* acc, uint16_t h)
{
    int e = (h >> 7) & 255;
    uint32_t m = h & 127u;
    if (e == 255) return; /* inf / NaN inputs are outside the contract */
    uint32_t M = (e == 0) ? m : (128u + m);
    int ee = (e == 0) ? 1 : e;
    /* x = M * 2^(ee-134), x^2 = M^2 * 2^(2ee-268) */
    big_add_shifted(acc, (uint64_t)M * M, 2 * ee);
}

static void add_f32_pos(big_t* acc, float v)
{
    /* v >= 0 finite: v = M * 2^(E) with the fp32 decomposition */
    uint32_t b = bits_of(v);
    int e = (int)((b >> 23) & 255u);
    uint32_t m = b & 0x7fffffu;
    if (e == 255 || (b >> 31)) return;
    uint32_t M = (e == 0) ? m : (m | 0x800000u);
    int ee = (e == 0) ? 1 : e;
    /* v = M * 2^(ee - 150); LSB 2^-268 -> position ee - 150 + 268 */
    big_add_shifted(acc, M, ee + 118);
}

float orc_exact_sumsq_bf16(const uint16_t* x, int64_t count, int64_t stride, float init)
{
    big_t acc;
    big_zero(&acc);
    if (init != 0.0f) add_f32_pos(&acc, init);
    for (int64_t t = 0; t < count; t++) add_sq_bf16(&acc, x[t * stride]);
    return big_to_f32_rn(&acc, 268);
}

void orc_importance(const uint16_t* X, int64_t T, int64_t K, int64_t ldx,
                    const float* I_in, float* I_out)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t k = 0; k < K; k++) {
        float init = I_in ? I_in[k] : 0.0f;
        I_out[k] = orc_exact_sumsq_bf16(X + k, T, ldx, init);
    }
}

/* ------------------------------------------------------------------------ */
/* R1: per-group absmax scale.  INT4: s = bf16_RN(fp32_RN(a / 7)).           */
/*     NVFP4: s = e4m3_RN_satfinite(a).  a = max |w| over the g weights.     */
/* R17: NVFP4 with a per-tensor fp32 scale gs = fp32_RN(amax / 448), amax    */
/*     the largest |w| of the tensor (gs = 0 when amax = 0); the stored     */
/*     group scale is s8 = e4m3_RN_satfinite(fp32_RN(a / gs)) (0 when       */
/*     gs = 0) and the group's effective scale is fp32_RN(gs * s8).  The    */
/*     largest group maps to the top of E4M3's range, so small weights keep */
/*     normal (4-significant-bit) scales instead of E4M3 subnormals.        */
/* ------------------------------------------------------------------------ */

float orc_global_scale(const uint16_t* W, int64_t N, int64_t K)
{
    float a = 0.0f;
    for (int64_t i = 0; i < N * K; i++) {
        float w = fabsf(orc_bf16_to_f32(W[i]));
        if (w > a) a = w;
    }
    return a > 0.0f ? a / 448.0f : 0.0f;
}

void orc_scales(const uint16_t* W, int64_t N, int64_t K, int fmt, int g, void* scales, float gs)
{
    int64_t G = K / g;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < N; r++) {
        for (int64_t j = 0; j < G; j++) {
            float a = 0.0f;
            for (int i = 0; i < g; i++) {
                float w = fabsf(orc_bf16_to_f32(W[r * K + j * g + i]));
                if (w > a) a = w;
            }
            if (fmt == ORC_INT4) {
                float d = a / 7.0f;
                ((uint16_t*)scales)[r * G + j] = orc_f32_to_bf16_rn(d);
            } else if (fmt == ORC_NVFP4) {
                ((uint8_t*)scales)[r * G + j] = orc_f32_to_e4m3_rn_sat(a);
            } else {
                ((uint8_t*)scales)[r * G + j] = gs > 0.0f ? orc_f32_to_e4m3_rn_sat(a / gs) : 0;
            }
        }
    }
}

/* Decoded magnitude of a stored scale; the sign bit (a choice tag) is
 * ignored.  For NVFP4 with a tensor scale this is the E4M3 factor s8. */
static float scale_value(const void* scales, int fmt, int64_t idx)
{
    if (fmt == ORC_INT4) return orc_bf16_to_f32(((const uint16_t*)scales)[idx] & 0x7fffu);
    return orc_e4m3_to_f32(((const uint8_t*)scales)[idx] & 0x7fu);
}

/* The scale that multiplies the codebook value: s itself, or fp32_RN(gs * s8)
 * with a tensor scale (R17). */
static float eff_scale(float s, int fmt, float gs)
{
    return fmt == ORC_NVFP4_GS ? gs * s : s;
}

/* R2: r = fp32_RN(1/s); u = fp32_RN(w * r).  A group is "live" when s > 0
 * and r is finite; every weight of a dead group has u = +0, choice 0 and no
 * share in any centroid. */
static int group_live(float s, float* r_out)
{
    if (!(s > 0.0f)) { *r_out = 0.0f; return 0; }
    float r = 1.0f / s;
    if (!isfinite(r)) { *r_out = 0.0f; return 0; }
    *r_out = r;
    return 1;
}

void orc_u(const uint16_t* W, int64_t N, int64_t K, int fmt, int g, const void* scales,
           float* u, float gs)
{
    int64_t G = K / g;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < N; r++) {
        for (int64_t k = 0; k < K; k++) {
            float s = scale_value(scales, fmt, r * G + k / g), rc;
            if (group_live(eff_scale(s, fmt, gs), &rc))
                u[r * K + k] = orc_bf16_to_f32(W[r * K + k]) * rc;
            else u[r * K + k] = 0.0f;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* R3: quantile initialisation (section 2, core mechanism 4, initialisation) */
/*     Sort all N*K values of u ascending (IEEE total order, so -0 < +0).    */
/*     T0_j = u_(floor((2j+1) M / 2n)), T1_j = u_(min(M-1, floor((j+1)M/n))) */
/* ------------------------------------------------------------------------ */

static uint32_t total_order_key(float f)
{
    uint32_t b = bits_of(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

static float key_to_f32(uint32_t k)
{
    return f32_of((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

static int cmp_u32(const void* a, const void* b)
{
    uint32_t x = *(const uint32_t*)a, y = *(const uint32_t*)b;
    return (x > y) - (x < y);
}

int64_t orc_rank_t0(int64_t M, int n, int j) { return (int64_t)(((u128)(2 * j + 1) * (u128)M) / (u128)(2 * n)); }
int64_t orc_rank_t1(int64_t M, int n, int j)
{
    int64_t r = (int64_t)(((u128)(j + 1) * (u128)M) / (u128)n);
    return r > M - 1 ? M - 1 : r;
}

int orc_init_codebooks(const uint16_t* W, int64_t N, int64_t K, int fmt, int g, void* scales,
                       float* T /* [2][16] */, float* gs_out /* NVFP4_GS: the tensor scale */)
{
    int64_t M = N * K;
    int n = (fmt == ORC_INT4) ? 16 : 15;
    float gs = fmt == ORC_NVFP4_GS ? orc_global_scale(W, N, K) : 0.0f;
    if (gs_out) *gs_out = gs;
    orc_scales(W, N, K, fmt, g, scales, gs);
    float* u = (float*)malloc(sizeof(float) * (size_t)M);
    uint32_t* key = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)M);
    if (!u || !key) { free(u); free(key); return 1; }
    orc_u(W, N, K, fmt, g, scales, u, gs);
    for (int64_t i = 0; i < M; i++) key[i] = total_order_key(u[i]);
    qsort(key, (size_t)M, sizeof(uint32_t), cmp_u32);
    for (int j = 0; j < 16; j++) {
        T[j] = 0.0f;
        T[16 + j] = 0.0f;
    }
    for (int j = 0; j < n; j++) {
        T[j] = key_to_f32(key[orc_rank_t0(M, n, j)]);
        T[16 + j] = key_to_f32(key[orc_rank_t1(M, n, j)]);
    }
    free(u);
    free(key);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* R4: assignment -- nearest entry, exact distances, lowest index on a tie   */
/*     (section 2, core mechanism 4, assign; 1-D Voronoi cells)              */
/* ------------------------------------------------------------------------ */

static int sub_exact_ok(float x, float y)
{
    if (x == 0.0f || y == 0.0f) return 1;
    int d = ilogbf(x) - ilogbf(y);
    return d <= 28 && d >= -28; /* then x - y needs at most 53 bits */
}

/* |u - t| as an exact big integer (units of 2^-149). */
static void big_absdiff(big_t* out, float u, float t)
{
    big_t bu, bt;
    int su = big_of_f32(&bu, u), st = big_of_f32(&bt, t);
    if (su != st) { big_addto(out, &bu, &bt); return; }
    if (big_cmp(&bu, &bt) >= 0) big_sub(out, &bu, &bt);
    else big_sub(out, &bt, &bu);
}

/* 1 when |u - a| < |u - b| exactly. */
static int closer(float u, float a, float b)
{
    if (sub_exact_ok(u, a) && sub_exact_ok(u, b)) {
        double da = fabs((double)u - (double)a), db = fabs((double)u - (double)b);
        return da < db;
    }
    big_t da, db;
    big_absdiff(&da, u, a);
    big_absdiff(&db, u, b);
    return big_cmp(&da, &db) < 0;
}

static int nearest(const float* T, int n, float u)
{
    int best = 0;
    for (int j = 1; j < n; j++)
        if (closer(u, T[j], T[best])) best = j;
    return best;
}

void orc_assign(const float* T, int n, const float* u, int64_t count, uint8_t* q)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++) q[i] = (uint8_t)nearest(T, n, u[i]);
}

/* Sort the first n entries ascending in IEEE total order (insertion sort). */
static void sort_codebook(float* t, int n)
{
    for (int i = 1; i < n; i++) {
        float v = t[i];
        uint32_t kv = total_order_key(v);
        int j = i - 1;
        while (j >= 0 && total_order_key(t[j]) > kv) { t[j + 1] = t[j]; j--; }
        t[j + 1] = v;
    }
}

/* ------------------------------------------------------------------------ */
/* R5: the per-group error and the codebook choice                           */
/*     (section 2, core mechanism 2: lower activation-weighted error wins)   */
/*     D_c = sum over the S weights of the group, ascending k, in fp64 with  */
/*     each operation rounded: e = u - T_c[q]; D += I_k * (e*e).             */
/*     choice = (D_1 < D_0), so T0 wins a tie.                               */
/* ------------------------------------------------------------------------ */

double orc_group_error(const float* u, const float* Ik, const float* Tc, const uint8_t* q, int S)
{
    double D = 0.0;
    for (int i = 0; i < S; i++) {
        double e = (double)u[i] - (double)Tc[q[i]];
        double e2 = e * e;
        double t = (double)Ik[i] * e2;
        D = D + t;
    }
    return D;
}

/* ------------------------------------------------------------------------ */
/* R6: refine -- activation-weighted centroid of each Voronoi cell           */
/*     (section 2, core mechanism 4, refine), in the normalised domain u:    */
/*       T_c[q] = sum A u / sum A over the cell, A = I_k * s^2,              */
/*     summed as exact integers: num += R_k(A 2^L u), den += R_k(A 2^L),     */
/*     where R_k rounds the exact product down (floor) in even columns k and */
/*     up (ceil) in odd columns -- no ties, no bias on average.              */
/*     L = B - E(I_max) - E(S2_max) - max(0, E(U_max)),                       */
/*     B = min(40, 61 - ceil(log2 M)), E(x) = frexp exponent (x < 2^E(x)).   */
/*     T = fp32(fp64(num) / fp64(den)) when den > 0, else unchanged; then the */
/*     codebook is re-sorted.                                                 */
/* ------------------------------------------------------------------------ */

/* floor(a * u) (up == 0) or ceil(a * u) (up != 0) of the exact product;
 * |result| < 2^62 assumed. */
int64_t orc_round_mul(double a, float u, int up)
{
    if (a == 0.0 || u == 0.0f) return 0;
    int ea, eu;
    double fa = frexp(a, &ea);
    float fu = frexpf(u, &eu);
    int64_t ma = (int64_t)ldexp(fa, 53); /* exact: |ma| < 2^53 */
    int64_t mu = (int64_t)ldexpf(fu, 24); /* exact: |mu| < 2^24 */
    int sh = (ea - 53) + (eu - 24);
    i128 p = (i128)ma * (i128)mu;
    int neg = p < 0;
    u128 m = neg ? (u128)(-p) : (u128)p;
    /* |a u| = m 2^sh; q = floor(|a u|), inexact = fractional part != 0 */
    u128 q;
    int inexact = 0;
    if (sh >= 0) {
        q = m << sh;
    } else {
        int rs = -sh;
        if (rs > 120) {
            q = 0;
            inexact = m != 0;
        } else {
            q = m >> rs;
            inexact = (m - (q << rs)) != 0;
        }
    }
    /* floor(x) = q for x >= 0, -q - inexact for x < 0; ceil mirrors it */
    int64_t v = (int64_t)q;
    if (!neg) return (up && inexact) ? v + 1 : v;
    return (!up && inexact) ? -v - 1 : -v;
}

static int clog2_i64(int64_t M)
{
    int c = 0;
    while (((int64_t)1 << c) < M) c++;
    return c;
}

int orc_fixed_point_L(int64_t M, double I_max, double S2_max, double U_max)
{
    int B = 61 - clog2_i64(M);
    if (B > 40) B = 40;
    if (!(I_max > 0.0) || !(S2_max > 0.0)) return 0;
    int eI, eS, eU = 0;
    frexp(I_max, &eI);
    frexp(S2_max, &eS);
    if (U_max > 0.0) frexp(U_max, &eU);
    if (eU < 0) eU = 0;
    return B - eI - eS - eU;
}

/* ------------------------------------------------------------------------ */
/* the fit (section 2, core mechanism 4: alternating optimisation)           */
/* ------------------------------------------------------------------------ */

typedef struct {
    int64_t near_ties;      /* groups with |D1-D0| < 1e-6 max(D0,D1), last iteration */
    int64_t groups_t1;      /* groups on T1, last iteration */
    int64_t empty_cells;    /* cells with den == 0 at the last refine (unfrozen books) */
    int64_t dead_groups;    /* groups with s == 0 or non-finite 1/s */
    int32_t L;              /* fixed-point exponent of the refine sums */
    int32_t pad;
} orc_stats;

typedef struct {
    const uint16_t* W;
    int64_t N, K;
    const float* I;
    const void* scales;
    int fmt, g, S, n;
    unsigned flags;
    float gs;  /* tensor scale (NVFP4_GS only) */
} layer_t;

/* One assign pass with codebooks T ([2][16]).  Fills per-group choice and
 * D of the chosen codebook (dead groups: choice 0, D 0), codes (q of the
 * chosen codebook) when non-NULL, near-tie count, and -- when bins is
 * non-NULL -- the fixed-point refine sums bins[c][q][0=num,1=den]. */
static void assign_pass(const layer_t* Ly, const float* T, int L, uint8_t* choice_out,
                        double* D_out, double* s2_out, uint8_t* codes, int64_t* near_ties,
                        int64_t bins[2][16][2])
{
    int64_t N = Ly->N, K = Ly->K, G = K / Ly->g, NS = K / Ly->S;
    int S = Ly->S, n = Ly->n;
    int64_t ties = 0;
    int64_t acc[2][16][2];
    memset(acc, 0, sizeof(acc));
#pragma omp parallel
    {
        int64_t my[2][16][2];
        memset(my, 0, sizeof(my));
        int64_t my_ties = 0;
        float* u = (float*)malloc(sizeof(float) * (size_t)S);
        float* Ik = (float*)malloc(sizeof(float) * (size_t)S);
        uint8_t* q0 = (uint8_t*)malloc((size_t)S);
        uint8_t* q1 = (uint8_t*)malloc((size_t)S);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < N; r++) {
            for (int64_t j = 0; j < NS; j++) {
                int64_t k0 = j * S;
                float s = scale_value(Ly->scales, Ly->fmt, r * G + k0 / Ly->g), rc;
                int live = group_live(eff_scale(s, Ly->fmt, Ly->gs), &rc);
                for (int i = 0; i < S; i++) {
                    u[i] = live ? orc_bf16_to_f32(Ly->W[r * K + k0 + i]) * rc : 0.0f;
                    Ik[i] = Ly->I[k0 + i];
                    q0[i] = (uint8_t)nearest(T, n, u[i]);
                    q1[i] = (uint8_t)nearest(T + 16, n, u[i]);
                }
                int c = 0;
                double Dc = 0.0;
                if (live) {
                    double D0 = orc_group_error(u, Ik, T, q0, S);
                    double D1 = orc_group_error(u, Ik, T + 16, q1, S);
                    if (!(Ly->flags & ORC_SINGLE_CODEBOOK)) c = (D1 < D0) ? 1 : 0;
                    double mx = D0 > D1 ? D0 : D1;
                    if (fabs(D1 - D0) < 1e-6 * mx) my_ties++;
                    Dc = c ? D1 : D0;
                }
                choice_out[r * NS + j] = (uint8_t)c;
                D_out[r * NS + j] = Dc;
                s2_out[r * NS + j] = live ? (double)s * (double)s : 0.0;
                const uint8_t* qc = c ? q1 : q0;
                if (codes) for (int i = 0; i < S; i++) codes[r * K + k0 + i] = qc[i];
                if (bins && live) {
                    double s2 = (double)s * (double)s;
                    for (int i = 0; i < S; i++) {
                        double A2L = ldexp((double)Ik[i] * s2, L); /* exact */
                        int up = (int)((k0 + i) & 1); /* column parity */
                        my[c][qc[i]][0] += orc_round_mul(A2L, u[i], up);
                        my[c][qc[i]][1] += orc_round_mul(A2L, 1.0f, up);
                    }
                }
            }
        }
#pragma omp critical
        {
            for (int c = 0; c < 2; c++)
                for (int q = 0; q < 16; q++) {
                    acc[c][q][0] += my[c][q][0];
                    acc[c][q][1] += my[c][q][1];
                }
            ties += my_ties;
        }
        free(u); free(Ik); free(q0); free(q1);
    }
    if (near_ties) *near_ties = ties;
    if (bins) memcpy(bins, acc, sizeof(acc));
}

/* Maxima that fix the refine's fixed-point exponent (exact). */
static void layer_maxima(const layer_t* Ly, double* I_max, double* S2_max, double* U_max,
                         int64_t* dead)
{
    int64_t N = Ly->N, K = Ly->K, G = K / Ly->g;
    double im = 0.0, sm = 0.0, um = 0.0;
    int64_t nd = 0;
    for (int64_t k = 0; k < K; k++) if ((double)Ly->I[k] > im) im = Ly->I[k];
    for (int64_t r = 0; r < N; r++) {
        for (int64_t j = 0; j < G; j++) {
            float s = scale_value(Ly->scales, Ly->fmt, r * G + j), rc;
            if (!group_live(eff_scale(s, Ly->fmt, Ly->gs), &rc)) { nd++; continue; }
            double s2 = (double)s * (double)s;
            if (s2 > sm) sm = s2;
            for (int i = 0; i < Ly->g; i++) {
                float u = orc_bf16_to_f32(Ly->W[r * K + j * Ly->g + i]) * rc;
                double a = fabs((double)u);
                if (a > um) um = a;
            }
        }
    }
    *I_max = im; *S2_max = sm; *U_max = um; *dead = nd;
}

int orc_fit(const uint16_t* W, int64_t N, int64_t K, const float* I, const void* scales,
            int fmt, int g, int S, int iters, unsigned flags, float* T /* [2][16] inout */,
            double* err_hist, orc_stats* st, float gs)
{
    layer_t Ly = { W, N, K, I, scales, fmt, g, S, (fmt == ORC_INT4) ? 16 : 15, flags, gs };
    int64_t NS = N * (K / S);
    uint8_t* choice = (uint8_t*)malloc((size_t)NS);
    double* D = (double*)malloc(sizeof(double) * (size_t)NS);
    double* s2 = (double*)malloc(sizeof(double) * (size_t)NS);
    if (!choice || !D || !s2) { free(choice); free(D); free(s2); return 1; }
    double I_max, S2_max, U_max;
    int64_t dead;
    layer_maxima(&Ly, &I_max, &S2_max, &U_max, &dead);
    int L = orc_fixed_point_L(N * K, I_max, S2_max, U_max);
    sort_codebook(T, Ly.n);
    sort_codebook(T + 16, Ly.n);
    orc_stats local;
    memset(&local, 0, sizeof(local));
    local.L = L;
    local.dead_groups = dead;
    for (int it = 0; it < iters; it++) {
        int64_t bins[2][16][2];
        int64_t ties = 0;
        assign_pass(&Ly, T, L, choice, D, s2, NULL, &ties, bins);
        double err = 0.0;
        int64_t nt1 = 0;
        for (int64_t i = 0; i < NS; i++) {
            err = err + s2[i] * D[i];
            nt1 += choice[i];
        }
        /* R17: the centroid weights and this sum use s8; the tensor scale is
         * common to every group and enters the objective as one factor. */
        err_hist[it] = fmt == ORC_NVFP4_GS ? err * ((double)gs * (double)gs) : err;
        local.near_ties = ties;
        local.groups_t1 = nt1;
        local.empty_cells = 0;
        for (int c = 0; c < 2; c++) {
            if (c == 0 && (flags & ORC_FREEZE_T0)) continue;
            if (c == 1 && (flags & ORC_FREEZE_T1)) continue;
            for (int j = 0; j < Ly.n; j++) {
                int64_t num = bins[c][j][0], den = bins[c][j][1];
                if (den > 0) T[c * 16 + j] = (float)((double)num / (double)den);
                else local.empty_cells++;
            }
            sort_codebook(T + c * 16, Ly.n);
        }
    }
    if (st) *st = local;
    free(choice); free(D); free(s2);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* R7: pack -- bf16 tables, final assign, 4-bit codes, tagged scales         */
/*     (section 2, core mechanism 3: BF16 codebooks, choice in sign bit;     */
/*      section 4: S=16 selection groups at 0.0625 bpw)                      */
/* ------------------------------------------------------------------------ */

int orc_pack(const uint16_t* W, int64_t N, int64_t K, const float* I, const void* scales,
             int fmt, int g, int S, unsigned flags, const float* T_in /* [2][16] */,
             uint16_t* T_bf16 /* [2][16] */, uint8_t* codes /* [N][K/2] */,
             void* scales_tagged /* like scales */, uint8_t* choice_bits /* [N][K/S/8] */,
             double* err_final, int64_t* near_ties, float gs)
{
    layer_t Ly = { W, N, K, I, scales, fmt, g, S, (fmt == ORC_INT4) ? 16 : 15, flags, gs };
    int64_t G = K / g, NS = K / S;
    float T[32], Tq[32];
    memcpy(T, T_in, sizeof(T));
    sort_codebook(T, Ly.n);
    sort_codebook(T + 16, Ly.n);
    for (int c = 0; c < 2; c++)
        for (int j = 0; j < 16; j++) {
            uint16_t h = (j < Ly.n) ? orc_f32_to_bf16_rn(T[c * 16 + j]) : 0;
            T_bf16[c * 16 + j] = h;
            Tq[c * 16 + j] = orc_bf16_to_f32(h);
        }
    uint8_t* choice = (uint8_t*)malloc((size_t)(N * NS));
    double* D = (double*)malloc(sizeof(double) * (size_t)(N * NS));
    double* s2 = (double*)malloc(sizeof(double) * (size_t)(N * NS));
    uint8_t* q = (uint8_t*)malloc((size_t)(N * K));
    if (!choice || !D || !s2 || !q) { free(choice); free(D); free(s2); free(q); return 1; }
    assign_pass(&Ly, Tq, 0, choice, D, s2, q, near_ties, NULL);
    for (int64_t r = 0; r < N; r++)
        for (int64_t k = 0; k < K; k += 2)
            codes[r * (K / 2) + k / 2] = (uint8_t)(q[r * K + k] | (q[r * K + k + 1] << 4));
    for (int64_t r = 0; r < N; r++)
        for (int64_t j = 0; j < G; j++) {
            int tag = (S == g) ? choice[r * NS + j] : 0;
            if (fmt == ORC_INT4) {
                uint16_t v = ((const uint16_t*)scales)[r * G + j] & 0x7fffu;
                ((uint16_t*)scales_tagged)[r * G + j] = (uint16_t)(v | (tag << 15));
            } else {
                uint8_t v = ((const uint8_t*)scales)[r * G + j] & 0x7fu;
                ((uint8_t*)scales_tagged)[r * G + j] = (uint8_t)(v | (tag << 7));
            }
        }
    if (S != g && choice_bits) {
        int64_t nb = (NS + 7) / 8;
        memset(choice_bits, 0, (size_t)(N * nb));
        for (int64_t r = 0; r < N; r++)
            for (int64_t j = 0; j < NS; j++)
                if (choice[r * NS + j]) choice_bits[r * nb + j / 8] |= (uint8_t)(1u << (j % 8));
    }
    /* err_final = sum over all weights, row-major, of I_k (w - s T[c][q])^2 */
    double err = 0.0;
    for (int64_t r = 0; r < N; r++)
        for (int64_t k = 0; k < K; k++) {
            float s = eff_scale(scale_value(scales, fmt, r * G + k / g), fmt, gs);
            int c = choice[r * NS + k / S];
            double wh = (double)s * (double)Tq[c * 16 + q[r * K + k]];
            double d = (double)orc_bf16_to_f32(W[r * K + k]) - wh;
            err = err + (double)I[k] * (d * d);
        }
    *err_final = err;
    free(choice); free(D); free(s2); free(q);
    return 0;
}

/* Per-weight dequantisation from the packed format (round-trip checks). */
void orc_unpack(const uint8_t* codes, const void* scales_tagged, const uint8_t* choice_bits,
                const uint16_t* T_bf16, int64_t N, int64_t K, int fmt, int g, int S,
                double* w_hat, uint8_t* choice_per_group /* [N][K/S] */, float gs)
{
    int64_t G = K / g, NS = K / S, nb = (NS + 7) / 8;
    for (int64_t r = 0; r < N; r++)
        for (int64_t k = 0; k < K; k++) {
            int64_t gi = r * G + k / g;
            int tag, c;
            float s;
            if (fmt == ORC_INT4) {
                uint16_t v = ((const uint16_t*)scales_tagged)[gi];
                tag = v >> 15;
                s = orc_bf16_to_f32(v & 0x7fffu);
            } else {
                uint8_t v = ((const uint8_t*)scales_tagged)[gi];
                tag = v >> 7;
                s = eff_scale(orc_e4m3_to_f32(v & 0x7fu), fmt, gs);
            }
            int64_t j = k / S;
            c = (S == g) ? tag : ((choice_bits[r * nb + j / 8] >> (j % 8)) & 1);
            if (k % S == 0) choice_per_group[r * NS + j] = (uint8_t)c;
            uint8_t byte = codes[r * (K / 2) + k / 2];
            int qv = (k & 1) ? (byte >> 4) : (byte & 15);
            w_hat[r * K + k] = (double)s * (double)orc_bf16_to_f32(T_bf16[c * 16 + qv]);
        }
}

/* ------------------------------------------------------------------------ */
/* R15: inference dequantisation (section 1: the dequantised values that    */
/*      decide the weights used at inference, W4A16; section 2 mech. 3:     */
/*      BF16 tables, choice in the scale's sign bit or in a bitmask).        */
/*      w_hat[n][k] = bf16_RN(s[n][k/g] * T_bf16[c][code[n][k]]): the exact  */
/*      product (at most 16 significant bits, exact in fp32) rounded once   */
/*      to the 16-bit activation type.  With a tensor scale (R17) s is the  */
/*      effective fp32 scale and the product is rounded to fp32 first:      */
/*      w_hat = bf16_RN(fp32_RN(fp32_RN(gs * s8) * T)).                      */
/* ------------------------------------------------------------------------ */
void orc_dequant_bf16(const uint8_t* codes, const void* scales_tagged, const uint8_t* choice_bits,
                      const uint16_t* T_bf16, int64_t N, int64_t K, int fmt, int g, int S,
                      uint16_t* w_hat, float gs)
{
    double* wd = (double*)malloc(sizeof(double) * (size_t)(N * K));
    uint8_t* ch = (uint8_t*)malloc((size_t)(N * (K / S)));
    orc_unpack(codes, scales_tagged, choice_bits, T_bf16, N, K, fmt, g, S, wd, ch, gs);
    for (int64_t i = 0; i < N * K; i++) w_hat[i] = orc_f32_to_bf16_rn((float)wd[i]);
    free(wd);
    free(ch);
}

/* W4A16 linear: Y[m][n] = sum_k X[m][k] * w_hat[n][k], summed in fp64 in k  */
/* order (X bf16 [M][ldx], w_hat bf16 [N][K]).                               */
void orc_linear(const uint16_t* X, int64_t M, int64_t ldx, const uint16_t* w_hat, int64_t N,
                int64_t K, double* Y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += (double)orc_bf16_to_f32(X[m * ldx + k]) *
                       (double)orc_bf16_to_f32(w_hat[n * K + k]);
            Y[m * N + n] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* AWQ-style pre-scaling ("Technical summary: AAAC", section 4: AAAC          */
/* combined with AWQ, which scales the weights before quantisation).  The    */
/* page gives no formula for the scaling; reading R16:                       */
/*   v_k  = I_k / tokens                      (fp64; the channel's mean x^2) */
/*   p_k  = v_k^(j/32), alpha = j/16 in [0, 1]: the product, in ascending i, */
/*          of v^(2^(i-5)) over the set bits i of j, each power taken by     */
/*          repeated fp64 square roots (v^(1/2), v^(1/4), ..., v^(1/32)), so */
/*          every step is a correctly rounded IEEE operation;                */
/*   z    = sqrt(max_k p_k * min_k p_k) over the live channels (I_k > 0);    */
/*   c_k  = fp32_RN(p_k / z) for live channels, 1 for dead ones;             */
/*   I'_k = fp32_RN(I_k / (c_k * c_k))        (fp64, c_k^2 exact);           */
/*   W'   = bf16_RN(fp32_RN(w * c_k)).                                       */
/* c scales the weights' input channels up where activations are large; the  */
/* activations of the scaled layer are x / c, whose energy is I'.            */
/* ------------------------------------------------------------------------ */
static double awq_power(double v, int j)
{
    double q[5];
    q[4] = sqrt(v);
    for (int i = 3; i >= 0; i--) q[i] = sqrt(q[i + 1]);
    double p = 1.0;
    for (int i = 0; i < 5; i++)
        if ((j >> i) & 1) p = p * q[i];
    return p;
}

void orc_awq_scales(const float* I, int64_t K, int64_t tokens, int j, float* c, float* I_out)
{
    double pmax = 0.0, pmin = 0.0;
    int any = 0;
    for (int64_t k = 0; k < K; k++) {
        if (!(I[k] > 0.0f)) continue;
        double p = awq_power((double)I[k] / (double)tokens, j);
        if (!any || p > pmax) pmax = p;
        if (!any || p < pmin) pmin = p;
        any = 1;
    }
    double z = any ? sqrt(pmax * pmin) : 1.0;
    for (int64_t k = 0; k < K; k++) {
        if (!(I[k] > 0.0f)) {
            c[k] = 1.0f;
            I_out[k] = I[k];
            continue;
        }
        double p = awq_power((double)I[k] / (double)tokens, j);
        c[k] = (float)(p / z);
        double cc = (double)c[k] * (double)c[k];
        I_out[k] = (float)((double)I[k] / cc);
    }
}

void orc_awq_scale_weights(const uint16_t* W, int64_t N, int64_t K, const float* c,
                           uint16_t* W_out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            float w = orc_bf16_to_f32(W[n * K + k]);
            float p = w * c[k];
            W_out[n * K + k] = orc_f32_to_bf16_rn(p);
        }
}
