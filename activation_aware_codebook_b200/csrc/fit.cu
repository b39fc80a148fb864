// fit.cu -- the alternating assign / refine fit and the 4-bit pack.
//
// "Technical summary: AAAC", section 2:
//   core mechanism 2  each weight group takes the codebook (T0 or T1) with the
//                     lower activation-weighted reconstruction error, weights
//                     I_k = sum_t X[t,k]^2;
//   core mechanism 3  BF16 codebooks; the choice rides in the sign bit of the
//                     positive scale (S == g) or in a bitmask (S < g, section 4);
//   core mechanism 4  alternating assign (nearest entry, Voronoi cells) and
//                     refine (activation-weighted centroid of each cell).
//
// One fit round = assign_pass<false> (one streaming pass over W) + fit_finalize
// (one block).  assign_pass: a warp covers 256 columns of a row (a 16-byte
// load per lane, 8 weights), keeps the codebook tables in shared memory,
// finds each weight's nearest entry in both codebooks by a branchless search
// over exact midpoint thresholds, sums the per-group errors in fp32 and
// reduces them over the group's lanes with shuffles.  A choice the fp32 sums
// cannot decide under their rounding-error bound is recomputed by the group's
// leader lane with the sequential fp64 rule.  The refine sums are exact
// integers, rint(A 2^L u) and rint(A 2^L) with A = I_k s^2, accumulated as
// 64-bit integers in shared-memory bins and flushed once per block, so the
// result does not depend on the order of the additions.
#include "common.cuh"
#include "internal.h"

namespace aaac {

struct FitCtl {
  float T[2][16];
  Books bk;
  int32_t n;
  int32_t L;
  double twoL;
  uint32_t Imax_bits;
  uint32_t Umax_bits;
  unsigned long long S2max_bits;
  unsigned long long dead_groups;
  unsigned long long bins[2][16][2];
  unsigned long long near_ties;
  unsigned long long groups_t1;
  unsigned long long exact_groups;
  unsigned long long empty_cells;
};

size_t fit_ctl_bytes() { return align256(sizeof(FitCtl)); }

size_t fit_ws_bytes(int64_t N, int64_t K) {
  const PassPlan pp = plan_pass(N, K);
  return fit_ctl_bytes() + align256((size_t)pp.blocks * sizeof(double));
}

size_t pack_extra_bytes(int64_t N, int64_t K, int S) {
  return align256((size_t)N * (size_t)(K / S));
}

// ---------------------------------------------------------------------------
// prep: the exact maxima that fix the refine's fixed-point exponent
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(kThreads)
fit_prep(const uint16_t* __restrict__ W, int N, int K, const float* __restrict__ I,
         const void* __restrict__ scales, int g, FitCtl* ctl, int ncb, int rows_per_chunk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // I_max over all columns
  uint32_t im = 0;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x)
    im = max(im, __float_as_uint(I[k]));
  const int cb = blockIdx.x % ncb, rc = blockIdx.x / ncb;
  const int col0 = cb * kSegCols + lane * 8;
  const bool active = col0 < K;
  const int lanes_g = g >> 3;
  const int G = K / g;
  uint32_t um = 0;
  double s2m = 0.0;
  unsigned long long dead = 0;
  const int r0 = rc * rows_per_chunk, r1 = min(N, r0 + rows_per_chunk);
  if (active) {
    for (int r = r0 + warp; r < r1; r += kWarps) {
      const float s = load_scale<FMT>(scales, (int64_t)r * G + col0 / g);
      float rcp;
      if (!scale_live(s, &rcp)) {
        if ((lane & (lanes_g - 1)) == 0) dead++;
        continue;
      }
      s2m = fmax(s2m, (double)s * (double)s);
      uint4 v = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)r * K + col0));
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const float wf = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
        um = max(um, __float_as_uint(fabsf(__fmul_rn(wf, rcp))));
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    im = max(im, __shfl_xor_sync(0xffffffffu, im, o));
    um = max(um, __shfl_xor_sync(0xffffffffu, um, o));
    s2m = fmax(s2m, __shfl_xor_sync(0xffffffffu, s2m, o));
    dead += __shfl_xor_sync(0xffffffffu, dead, o);
  }
  if (lane == 0) {
    if (im) atomicMax(&ctl->Imax_bits, im);
    if (um) atomicMax(&ctl->Umax_bits, um);
    if (s2m > 0.0) atomicMax(&ctl->S2max_bits, (unsigned long long)__double_as_longlong(s2m));
    if (dead) atomicAdd(&ctl->dead_groups, dead);
  }
}

__device__ inline int frexp_exponent(double x) {
  int e;
  frexp(x, &e);
  return e;
}

__device__ void write_stats(const FitCtl* ctl, aaac_stats* st) {
  if (!st) return;
  st->near_ties = (int64_t)ctl->near_ties;
  st->groups_t1 = (int64_t)ctl->groups_t1;
  st->empty_cells = (int64_t)ctl->empty_cells;
  st->dead_groups = (int64_t)ctl->dead_groups;
  st->exact_groups = (int64_t)ctl->exact_groups;
  st->L = ctl->L;
  st->reserved = 0;
}

// L = B - E(I_max) - E(S2_max) - max(0, E(U_max)), B = min(40, 61 - ceil(log2 M))
__global__ void fit_setup(FitCtl* ctl, float* T_user, int64_t M, int n, aaac_stats* st) {
  if (threadIdx.x != 0) return;
  int c = 0;
  while (((int64_t)1 << c) < M) c++;
  int B = 61 - c;
  if (B > 40) B = 40;
  const double Imax = (double)__uint_as_float(ctl->Imax_bits);
  const double S2max = __longlong_as_double((long long)ctl->S2max_bits);
  const double Umax = (double)__uint_as_float(ctl->Umax_bits);
  int L = 0;
  if (Imax > 0.0 && S2max > 0.0) {
    int eU = Umax > 0.0 ? frexp_exponent(Umax) : 0;
    if (eU < 0) eU = 0;
    L = B - frexp_exponent(Imax) - frexp_exponent(S2max) - eU;
  }
  ctl->L = L;
  ctl->twoL = ldexp(1.0, L);
  ctl->n = n;
  for (int b = 0; b < 2; b++) {
    for (int j = 0; j < 16; j++) ctl->T[b][j] = T_user[b * 16 + j];
    sort_book(ctl->T[b], n);
    build_book(ctl->T[b], n, &ctl->bk.b[b]);
    for (int j = 0; j < 16; j++) T_user[b * 16 + j] = ctl->T[b][j];
  }
  write_stats(ctl, st);
}

// ---------------------------------------------------------------------------
// the streaming assign pass (fit: + refine sums; pack: + outputs)
// ---------------------------------------------------------------------------
struct PackOut {
  uint8_t* codes;
  void* tagged;
  uint8_t* choice_bytes;
};

template <int FMT, bool PACK>
__global__ void __launch_bounds__(kThreads, 2)
assign_pass(const uint16_t* __restrict__ W, int N, int K, const float* __restrict__ I,
            const void* __restrict__ scales, int g, int S, uint32_t flags, FitCtl* ctl,
            double* __restrict__ errp, int ncb, int rows_per_chunk, float tau, PackOut po) {
  __shared__ Books sbk;
  __shared__ unsigned long long sbins[64];
  __shared__ double sred[kThreads];
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&ctl->bk);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&sbk);
    for (int i = threadIdx.x; i < (int)(sizeof(Books) / 4); i += blockDim.x) dst[i] = src[i];
    if (!PACK && threadIdx.x < 64) sbins[threadIdx.x] = 0ull;
  }
  const double twoL = ctl->twoL;
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = blockIdx.x % ncb, rc = blockIdx.x / ncb;
  const int col0 = cb * kSegCols + lane * 8;
  const bool active = col0 < K;
  const int G = K / g, KS = K / S;
  const int lanes_s = S >> 3, lanes_g = g >> 3;
  const int leader_lane = lane & ~(lanes_s - 1);
  const bool s_leader = lane == leader_lane;
  const bool single = (flags & AAAC_SINGLE_CODEBOOK) != 0;

  float Ik[8];
  double I2L[8];
  if (active) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(I + col0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(I + col0 + 4));
    Ik[0] = a.x; Ik[1] = a.y; Ik[2] = a.z; Ik[3] = a.w;
    Ik[4] = b.x; Ik[5] = b.y; Ik[6] = b.z; Ik[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++) Ik[i] = 0.0f;
  }
#pragma unroll
  for (int i = 0; i < 8; i++) I2L[i] = (double)Ik[i] * twoL;

  double err_acc = 0.0;
  unsigned long long n_near = 0, n_exact = 0, n_t1 = 0;
  const int r0 = rc * rows_per_chunk, r1 = min(N, r0 + rows_per_chunk);
  for (int r = r0 + warp; r < r1; r += kWarps) {  // warp-uniform trip count
    uint4 v = make_uint4(0, 0, 0, 0);
    float s = 0.0f;
    if (active) {
      v = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)r * K + col0));
      s = load_scale<FMT>(scales, (int64_t)r * G + col0 / g);
    }
    float rcp;
    const bool live = active && scale_live(s, &rcp);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float u[8], t0v[8], t1v[8];
    int q0[8], q1[8];
    float d0 = 0.0f, d1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float wf = (i & 1) ? bf16_hi(wv[i >> 1]) : bf16_lo(wv[i >> 1]);
      u[i] = live ? __fmul_rn(wf, rcp) : 0.0f;
      const int c0 = book_count(sbk.b[0], u[i]);
      const int c1 = book_count(sbk.b[1], u[i]);
      q0[i] = sbk.b[0].idx[c0];
      q1[i] = sbk.b[1].idx[c1];
      t0v[i] = sbk.b[0].val[c0];
      t1v[i] = sbk.b[1].val[c1];
      const float e0 = __fsub_rn(u[i], t0v[i]);
      const float e1 = __fsub_rn(u[i], t1v[i]);
      d0 = __fmaf_rn(Ik[i], __fmul_rn(e0, e0), d0);
      d1 = __fmaf_rn(Ik[i], __fmul_rn(e1, e1), d1);
    }
    for (int o = 1; o < lanes_s; o <<= 1) {
      d0 = __fadd_rn(d0, __shfl_xor_sync(0xffffffffu, d0, o));
      d1 = __fadd_rn(d1, __shfl_xor_sync(0xffffffffu, d1, o));
    }
    // The choice (section 2, core mechanism 2): decided in fp32 when the gap
    // exceeds the fp32 error bound, else by the sequential fp64 rule.
    int choice = 0;
    bool exact = false;
    if (live && !single) {
      const float sum = __fadd_rn(d0, d1);
      const float gap = fabsf(__fsub_rn(d1, d0));
      const bool decided = (sum >= 8.673617379884035e-19f) && (sum < 3.0e38f) &&
                           (gap > __fmul_rn(tau, sum));
      if (decided) choice = (d1 < d0) ? 1 : 0;
      else exact = true;
    }
    double E0 = 0.0, E1 = 0.0;
    if (exact && s_leader) {
      const int kbase = col0 - (lane - leader_lane) * 8;  // first column of the group
      const uint16_t* wrow = W + (int64_t)r * K + kbase;
      for (int j = 0; j < S; j++) {
        const float wf = __uint_as_float((uint32_t)wrow[j] << 16);
        const float uj = __fmul_rn(wf, rcp);
        const double Ij = (double)I[kbase + j];
        const double ea = __dsub_rn((double)uj, (double)sbk.b[0].val[book_count(sbk.b[0], uj)]);
        const double eb = __dsub_rn((double)uj, (double)sbk.b[1].val[book_count(sbk.b[1], uj)]);
        E0 = __dadd_rn(E0, __dmul_rn(Ij, __dmul_rn(ea, ea)));
        E1 = __dadd_rn(E1, __dmul_rn(Ij, __dmul_rn(eb, eb)));
      }
      choice = (E1 < E0) ? 1 : 0;
    }
    choice = __shfl_sync(0xffffffffu, choice, leader_lane);

    if (s_leader && live) {
      double D0 = exact ? E0 : (double)d0, D1 = exact ? E1 : (double)d1;
      if (single) D1 = D0 + fabs(D0) + 1.0;  // no near-tie count when T1 is off
      const double mx = fmax(D0, D1);
      if (fabs(D1 - D0) < 1e-6 * mx) n_near++;
      n_exact += exact ? 1 : 0;
      n_t1 += choice;
      if (!PACK) err_acc += (double)s * (double)s * (choice ? D1 : D0);
    }

    if (!PACK) {
      if (live) {
        const double s2 = (double)s * (double)s;
#pragma unroll
        for (int i = 0; i < 8; i++) {
          const int q = choice ? q1[i] : q0[i];
          const double A = __dmul_rn(I2L[i], s2);  // exact: 24 + 16 bits
          const double num = __dsub_rn(__fma_rn(A, (double)u[i], kMagic), kMagic);
          const double den = __dsub_rn(__dadd_rn(A, kMagic), kMagic);
          atomicAdd(&sbins[(choice * 16 + q) * 2 + 0], (unsigned long long)(long long)num);
          atomicAdd(&sbins[(choice * 16 + q) * 2 + 1], (unsigned long long)(long long)den);
        }
      }
    } else if (active) {
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int q = choice ? q1[i] : q0[i];
        packed |= (uint32_t)q << (4 * i);
        const float wf = (i & 1) ? bf16_hi(wv[i >> 1]) : bf16_lo(wv[i >> 1]);
        const double wh = (double)s * (double)(choice ? t1v[i] : t0v[i]);
        const double d = __dsub_rn((double)wf, wh);
        err_acc = __fma_rn((double)Ik[i], __dmul_rn(d, d), err_acc);
      }
      *reinterpret_cast<uint32_t*>(po.codes + ((int64_t)r * K + col0) / 2) = packed;
      if ((lane & (lanes_g - 1)) == 0) {
        const int64_t gi = (int64_t)r * G + col0 / g;
        const uint32_t tag = (S == g) ? (uint32_t)choice : 0u;
        if (FMT == kInt4) {
          const uint32_t h = reinterpret_cast<const unsigned short*>(scales)[gi];
          reinterpret_cast<unsigned short*>(po.tagged)[gi] =
              (unsigned short)((h & 0x7fffu) | (tag << 15));
        } else {
          const uint32_t b = reinterpret_cast<const unsigned char*>(scales)[gi];
          reinterpret_cast<unsigned char*>(po.tagged)[gi] = (unsigned char)((b & 0x7fu) | (tag << 7));
        }
      }
      if (S != g && s_leader) po.choice_bytes[(int64_t)r * KS + col0 / S] = (uint8_t)choice;
    }
  }

  // fixed-order block reduction of the error partials
  sred[threadIdx.x] = err_acc;
  for (int o = 16; o > 0; o >>= 1) {
    n_near += __shfl_xor_sync(0xffffffffu, n_near, o);
    n_exact += __shfl_xor_sync(0xffffffffu, n_exact, o);
    n_t1 += __shfl_xor_sync(0xffffffffu, n_t1, o);
  }
  if (lane == 0) {
    if (n_near) atomicAdd(&ctl->near_ties, n_near);
    if (n_exact) atomicAdd(&ctl->exact_groups, n_exact);
    if (n_t1) atomicAdd(&ctl->groups_t1, n_t1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < kThreads; i++) t = __dadd_rn(t, sred[i]);
    errp[blockIdx.x] = t;
  }
  if (!PACK && threadIdx.x < 64) {
    const unsigned long long b = sbins[threadIdx.x];
    if (b) atomicAdd(&ctl->bins[0][0][0] + threadIdx.x, b);
  }
}

// refine (section 2, core mechanism 4): T = fp32(fp64(num) / fp64(den)) when
// den > 0, else unchanged; then sort and rebuild the tables.
__global__ void fit_finalize(FitCtl* ctl, const double* __restrict__ errp, int nblocks,
                             double* err_hist, int it, uint32_t flags, float* T_user,
                             aaac_stats* st) {
  if (threadIdx.x != 0) return;
  double e = 0.0;
  for (int b = 0; b < nblocks; b++) e = __dadd_rn(e, errp[b]);
  if (err_hist) err_hist[it] = e;
  const int n = ctl->n;
  unsigned long long empty = 0;
  for (int c = 0; c < 2; c++) {
    const bool frozen = (c == 0) ? (flags & AAAC_FREEZE_T0) : (flags & AAAC_FREEZE_T1);
    if (frozen) continue;
    for (int j = 0; j < n; j++) {
      const long long num = (long long)ctl->bins[c][j][0];
      const long long den = (long long)ctl->bins[c][j][1];
      if (den > 0)
        ctl->T[c][j] = __double2float_rn(__ddiv_rn(__ll2double_rn(num), __ll2double_rn(den)));
      else
        empty++;
    }
    sort_book(ctl->T[c], n);
    build_book(ctl->T[c], n, &ctl->bk.b[c]);
  }
  ctl->empty_cells = empty;
  for (int c = 0; c < 2; c++)
    for (int j = 0; j < 16; j++) T_user[c * 16 + j] = ctl->T[c][j];
  write_stats(ctl, st);
  for (int i = 0; i < 64; i++) (&ctl->bins[0][0][0])[i] = 0ull;
  ctl->near_ties = 0;
  ctl->groups_t1 = 0;
}

static float choice_tau(int S) {
  int lg = 0;
  while ((8 << lg) < S) lg++;
  return (float)((12 + lg) * ldexp(1.0, -22));
}

template <int FMT>
static void launch_fit_t(const uint16_t* W, int64_t N, int64_t K, const float* I,
                         const void* scales, int g, int S, int iters, uint32_t flags, float* T,
                         double* err_hist, aaac_stats* stats, void* ws, cudaStream_t st) {
  const PassPlan pp = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  double* errp = reinterpret_cast<double*>(reinterpret_cast<char*>(ws) + fit_ctl_bytes());
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pp.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl, pp.ncb,
                                                pp.rows_per_chunk);
  fit_setup<<<1, 32, 0, st>>>(ctl, T, N * K, ncodes(FMT), stats);
  const float tau = choice_tau(S);
  for (int it = 0; it < iters; it++) {
    assign_pass<FMT, false><<<pp.blocks, kThreads, 0, st>>>(
        W, (int)N, (int)K, I, scales, g, S, flags, ctl, errp, pp.ncb, pp.rows_per_chunk, tau,
        PackOut{nullptr, nullptr, nullptr});
    fit_finalize<<<1, 32, 0, st>>>(ctl, errp, pp.blocks, err_hist, it, flags, T, stats);
  }
  count_launches(2 + 2 * iters);
}

cudaError_t launch_fit(const uint16_t* W, int64_t N, int64_t K, const float* I,
                       const void* scales, int fmt, int g, int S, int iters, uint32_t flags,
                       float* T, double* err_hist, aaac_stats* stats, void* ws, cudaStream_t st) {
  if (fmt == kInt4)
    launch_fit_t<kInt4>(W, N, K, I, scales, g, S, iters, flags, T, err_hist, stats, ws, st);
  else
    launch_fit_t<kNvfp4>(W, N, K, I, scales, g, S, iters, flags, T, err_hist, stats, ws, st);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// pack
// ---------------------------------------------------------------------------
__global__ void pack_setup(FitCtl* ctl, const float* T_user, int n, uint16_t* T_bf16) {
  if (threadIdx.x != 0) return;
  ctl->n = n;
  for (int b = 0; b < 2; b++) {
    float t[16];
    for (int j = 0; j < 16; j++) t[j] = T_user[b * 16 + j];
    sort_book(t, n);
    for (int j = 0; j < 16; j++) {
      const unsigned short h = j < n ? __bfloat16_as_ushort(__float2bfloat16_rn(t[j])) : 0;
      T_bf16[b * 16 + j] = h;
      ctl->T[b][j] = __uint_as_float((uint32_t)h << 16);
    }
    build_book(ctl->T[b], n, &ctl->bk.b[b]);
  }
}

__global__ void pack_finalize(const double* __restrict__ errp, int nblocks, double* err_final) {
  if (threadIdx.x != 0) return;
  double e = 0.0;
  for (int b = 0; b < nblocks; b++) e = __dadd_rn(e, errp[b]);
  if (err_final) *err_final = e;
}

// choice bytes [N][K/S] -> bits [N][ceil(K/S/8)], LSB first
__global__ void pack_bits(const uint8_t* __restrict__ cb, int64_t N, int KS, uint8_t* bits) {
  const int nb = (KS + 7) / 8;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N * nb) return;
  const int64_t r = i / nb;
  const int j0 = (int)(i % nb) * 8;
  uint32_t byte = 0;
  for (int j = 0; j < 8 && j0 + j < KS; j++) byte |= (uint32_t)(cb[r * KS + j0 + j] & 1u) << j;
  bits[i] = (uint8_t)byte;
}

cudaError_t launch_pack(const uint16_t* W, int64_t N, int64_t K, const float* I,
                        const void* scales, int fmt, int g, int S, uint32_t flags, const float* T,
                        uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                        uint8_t* choice_bits, double* err_final, void* ws, cudaStream_t st) {
  const PassPlan pp = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  double* errp = reinterpret_cast<double*>(reinterpret_cast<char*>(ws) + fit_ctl_bytes());
  uint8_t* cbytes = reinterpret_cast<uint8_t*>(ws) + fit_ws_bytes(N, K);
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  pack_setup<<<1, 32, 0, st>>>(ctl, T, ncodes(fmt), T_bf16);
  const float tau = choice_tau(S);
  const PackOut po{codes, scales_tagged, cbytes};
  if (fmt == kInt4)
    assign_pass<kInt4, true><<<pp.blocks, kThreads, 0, st>>>(
        W, (int)N, (int)K, I, scales, g, S, flags, ctl, errp, pp.ncb, pp.rows_per_chunk, tau, po);
  else
    assign_pass<kNvfp4, true><<<pp.blocks, kThreads, 0, st>>>(
        W, (int)N, (int)K, I, scales, g, S, flags, ctl, errp, pp.ncb, pp.rows_per_chunk, tau, po);
  pack_finalize<<<1, 32, 0, st>>>(errp, pp.blocks, err_final);
  if (S != g) {
    const int KS = (int)(K / S);
    const int64_t total = N * ((KS + 7) / 8);
    pack_bits<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(cbytes, N, KS, choice_bits);
  }
  count_launches(S != g ? 4 : 3);
  return cudaGetLastError();
}

}  // namespace aaac
