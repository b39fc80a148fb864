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
// One fit round is ONE launch of fit_pass<false>: a streaming pass over W whose
// last block to finish (atomic ticket, no waiting) does the refine, sorts the
// books, rebuilds the tables and records the error.  Per block: 2 warps; a warp
// covers 256 columns of a row (16 bytes per lane) and walks the rows of its
// chunk with a 3-deep cp.async ring, so several rows per warp are in flight.
// The grid is one wave (10 blocks per SM).
//
// Nearest entry in both books at once (exact):
//   the midpoint thresholds of both books, merged and deduplicated (at most
//   30), split the u line into merged cells; cell m fixes both books' nearest
//   entries, mval[m] = (v0, v1).  bucket b = rint(u * la + 64) (one FFMA);
//   mlut[b] = the number c of merged thresholds at or below every u of the
//   bucket (kCrowded when two or more fall inside it: a binary search takes
//   over);
//   then m = c + (u >= mthr[c]) -- exact, because every threshold is the
//   smallest fp32 above an exact midpoint.
// Choice: fp32 group sums when their gap exceeds the rounding bound, else the
//   sequential fp64 rule (the group's leader lane recomputes it).
// Refine sums: per weight rint(A 2^L u) and rint(A 2^L), A = I_k s^2, as the
//   raw bit patterns of fp64 FMA/ADD results with magic constants; summed in
//   shared-memory bins modulo 2^64, which keeps num exact modulo 2^51 and den
//   modulo 2^52 -- exact because every bin's partial sum stays far below those
//   bounds.  Each pair of lanes owns one set of bins and the two lanes update it
//   in turn (read-modify-write, no atomics); halving the bins' shared memory
//   lets 16 warps share an SM.  Integer sums make the result order-free.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace aaac {

constexpr int kNB = 128;                  // bucket LUT entries
constexpr int kFitWarps = 2;
constexpr int kFitThreads = kFitWarps * 32;
constexpr int kStages = 3;                // rows per warp in flight
constexpr int kFitBlocksPerSM = 10;
constexpr float kBucketMagic = 12582912.0f;           // 1.5 * 2^23
constexpr double kDenMagic = 4503599627370496.0;      // 2^52
#define kInf __int_as_float(0x7f800000)

// Merged tables of both books (see the header comment).  Entries past the
// last cell are padding (mthr = +inf); 33 entries keep every lookup in bounds.
constexpr int kMerged = 33;
constexpr uint32_t kCrowded = 31;  // lut value of a crowded bucket (base counts are <= 30)
struct Tables {
  Book bk[2];
  float mthr[kMerged];     // merged thresholds, ascending, +inf padded
  float2 mval[kMerged];    // (v0[count0], v1[count1]) of merged cell m
  uint8_t mcell[kMerged];  // count0 | count1 << 4 of merged cell m
  uint8_t mlut[kNB];       // bucket -> merged base count, kCrowded = crowded bucket
  float la;
  int32_t nm;              // number of merged thresholds
  int32_t pad[2];
};

struct FitCtl {
  Tables tb;
  float T[2][16];
  int32_t n;
  int32_t L;
  double twoL;
  uint32_t Imax_bits;
  uint32_t Umax_bits;
  unsigned long long S2max_bits;
  unsigned long long dead_groups;
  long long bins[2][16][2];
  unsigned long long near_ties;
  unsigned long long groups_t1;
  unsigned long long exact_groups;
  unsigned long long empty_cells;
  unsigned int ticket;
  int32_t pad2;
};

size_t fit_ctl_bytes() { return align256(sizeof(FitCtl)); }

static PassPlan fit_plan(int64_t N, int64_t K) { return plan_pass(N, K, 148 * kFitBlocksPerSM); }

size_t fit_ws_bytes(int64_t N, int64_t K) {
  const PassPlan pp = fit_plan(N, K);
  return fit_ctl_bytes() + align256((size_t)pp.blocks * sizeof(double));
}

size_t pack_extra_bytes(int64_t N, int64_t K, int S) {
  return align256((size_t)N * (size_t)(K / S));
}

static size_t smem_bytes(bool pack) {
  size_t b = (sizeof(Tables) + 15) & ~(size_t)15;
  b += (size_t)kFitWarps * kStages * 32 * sizeof(uint4);
  if (!pack) b += (size_t)kFitWarps * 32 * 16 * sizeof(ulonglong2);
  return b;
}

// ---------------------------------------------------------------------------
// buckets and tables
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bucket_t(float u, float la) {
  return __fmaf_rn(u, la, kBucketMagic + (float)(kNB / 2));
}

// rint(x * la + 64) without wrap-around, clamped to [-1, kNB] (table builder).
__device__ inline int bucket_raw(float x, float la) {
  if (!(fabsf(x) * la < 4.0e6f)) return (x < 0.0f) ? -1 : kNB;
  const int r = (int)(__float_as_uint(bucket_t(x, la)) - __float_as_uint(kBucketMagic));
  return min(max(r, -1), kNB);
}

// Merge both books' thresholds (one thread).
__device__ void merge_thresholds(Tables& tb) {
  const Book& a = tb.bk[0];
  const Book& b = tb.bk[1];
  int i = 0, j = 0, n = 0;
  const int na = a.m - 1, nb = b.m - 1;
  while (i < na || j < nb) {
    float t;
    if (j >= nb || (i < na && a.thr[i] < b.thr[j])) t = a.thr[i++];
    else if (i >= na || b.thr[j] < a.thr[i]) t = b.thr[j++];
    else { t = a.thr[i++]; j++; }  // equal thresholds: one cell boundary
    tb.mthr[n++] = t;
  }
  tb.nm = n;
  for (int k = n; k < kMerged; k++) tb.mthr[k] = kInf;
}

// Cell m of the merged tables (thread per cell).
__device__ void merged_cell(Tables& tb, int m) {
  int c0 = 0, c1 = 0;
  if (m >= 1 && m <= tb.nm) {
    const float lo = tb.mthr[m - 1];  // smallest u of the cell
    for (int i = 0; i + 1 < tb.bk[0].m; i++) c0 += (tb.bk[0].thr[i] <= lo) ? 1 : 0;
    for (int i = 0; i + 1 < tb.bk[1].m; i++) c1 += (tb.bk[1].thr[i] <= lo) ? 1 : 0;
  }
  tb.mcell[m] = (uint8_t)(c0 | (c1 << 4));
  tb.mval[m] = make_float2(tb.bk[0].val[c0], tb.bk[1].val[c1]);
}

// All tables from the codebooks sT[2][16] (shared memory), by every thread of
// one block (blockDim >= 64): sort (optional), distinct values, exact midpoint
// thresholds, merged thresholds, merged cells, and the bucket table (bucket b
// counts the merged thresholds at or below its smallest u, or kCrowded when
// two or more fall strictly inside it).
__device__ void build_tables(Tables& tb, float (*sT)[16], int n, bool sort_first) {
  __shared__ int s_rb[32], s_first[32];
  const int tid = threadIdx.x;
  if (tid < 2) {
    const int c = tid;
    if (sort_first) sort_book(sT[c], n);
    Book& bk = tb.bk[c];
    int m = 0;
    for (int j = 0; j < n; j++) {
      if (m == 0 || !(sT[c][j] == bk.val[m - 1])) {  // -0 == +0: one value
        bk.val[m] = sT[c][j];
        bk.idx[m] = j;
        m++;
      }
    }
    for (int i = m; i < 16; i++) { bk.val[i] = bk.val[m - 1]; bk.idx[i] = bk.idx[m - 1]; }
    bk.m = m;
  }
  __syncthreads();
  if (tid < 32) {
    Book& bk = tb.bk[tid >> 4];
    const int i = tid & 15;
    bk.thr[i] = (i + 1 < bk.m) ? midpoint_threshold(bk.val[i], bk.val[i + 1]) : kInf;
  }
  __syncthreads();
  if (tid == 0) merge_thresholds(tb);
  __syncthreads();
  if (tid < tb.nm) {
    const float th = tb.mthr[tid];
    const int rb = bucket_raw(th, tb.la);
    s_rb[tid] = rb;
    s_first[tid] = bucket_raw(nextafterf(th, -kInf), tb.la) < rb;  // th opens its bucket
  }
  __syncthreads();
  for (int m = tid; m < kMerged; m += blockDim.x) merged_cell(tb, m);
  for (int b = tid; b < kNB; b += blockDim.x) {
    int base = 0, inner = 0;
    for (int i = 0; i < tb.nm; i++) {
      const int rb = s_rb[i];
      if (rb < b || (rb == b && s_first[i])) base++;
      else if (rb == b) inner++;
    }
    tb.mlut[b] = (uint8_t)(inner > 1 ? kCrowded : base);
  }
  __syncthreads();
}

__device__ void store_tables(FitCtl* ctl, const Tables& tb) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(&tb);
  uint32_t* dst = reinterpret_cast<uint32_t*>(&ctl->tb);
  for (int i = threadIdx.x; i < (int)(sizeof(Tables) / 4); i += blockDim.x) dst[i] = src[i];
}

// ---------------------------------------------------------------------------
// prep: the exact maxima that fix the refine's fixed-point exponent and the
// bucket scale
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(kThreads)
fit_prep(const uint16_t* __restrict__ W, int N, int K, const float* __restrict__ I,
         const void* __restrict__ scales, int g, FitCtl* ctl, int ncb, int rows_per_chunk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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

__device__ float bucket_scale(const FitCtl* ctl) {
  const float Umax = __uint_as_float(ctl->Umax_bits);
  return Umax > 0.0f ? __fdiv_rn(62.5f, Umax) : 0.0f;  // |u| * la < 63: buckets 1..127
}

// L = B - E(I_max) - E(S2_max) - max(0, E(U_max)), B = min(40, 61 - ceil(log2 M))
__global__ void __launch_bounds__(kFitThreads)
fit_setup(FitCtl* ctl, float* T_user, int64_t M, int n, aaac_stats* st) {
  __shared__ Tables tb;
  if (threadIdx.x == 0) {
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
    tb.la = bucket_scale(ctl);
  }
  __shared__ float sT[2][16];
  if (threadIdx.x < 32) sT[threadIdx.x >> 4][threadIdx.x & 15] = T_user[threadIdx.x];
  __syncthreads();
  build_tables(tb, sT, n, true);
  store_tables(ctl, tb);
  if (threadIdx.x < 32) {
    const float t = sT[threadIdx.x >> 4][threadIdx.x & 15];
    ctl->T[threadIdx.x >> 4][threadIdx.x & 15] = t;
    T_user[threadIdx.x] = t;
  }
  if (threadIdx.x == 0) write_stats(ctl, st);
}

// ---------------------------------------------------------------------------
// the streaming pass (fit: + refine sums; pack: + outputs)
// ---------------------------------------------------------------------------
struct PackOut {
  uint8_t* codes;
  void* tagged;
  uint8_t* choice_bytes;
  double* err_final;
};

struct RoundOut {
  double* err_hist;
  float* T_user;
  aaac_stats* stats;
  int it;
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Packed pairs of fp32 (Blackwell f32x2 arithmetic, each lane rounded to nearest).
__device__ __forceinline__ unsigned long long f2pack(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2unpack(unsigned long long p) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(p));
  return make_float2(a, b);
}
__device__ __forceinline__ unsigned long long f2sub(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long f2mul(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// The refine of one round, run by the last block of the pass: centroids from
// the integer sums (section 2, core mechanism 4), T = fp32(fp64(num) /
// fp64(den)) when den > 0, else unchanged; then sorted books and new tables.
// Everything is staged in shared memory and spread over the block's threads.
__device__ void round_finalize(FitCtl* ctl, Tables& tb, const double* errp, int nb,
                               uint32_t flags, const RoundOut& ro, double* sred) {
  __shared__ float sT[2][16];
  __shared__ long long sb[64];
  __shared__ int s_upd[2];
  const int tid = threadIdx.x;
  double part = 0.0;
  for (int b = tid; b < nb; b += blockDim.x) part = __dadd_rn(part, __ldcg(errp + b));
  sred[tid] = part;
  if (tid < 64) sb[tid] = __ldcg(&ctl->bins[0][0][0] + tid);
  if (tid < 32) sT[tid >> 4][tid & 15] = ctl->T[tid >> 4][tid & 15];
  if (tid < 2) s_upd[tid] = 0;
  __syncthreads();
  if (tid == 0) {
    double e = 0.0;
    for (int i = 0; i < (int)blockDim.x; i++) e = __dadd_rn(e, sred[i]);
    if (ro.err_hist) ro.err_hist[ro.it] = e;
  }
  const int n = ctl->n;
  if (tid < 32) {
    const int c = tid >> 4, j = tid & 15;
    const bool frozen = (c == 0) ? (flags & AAAC_FREEZE_T0) : (flags & AAAC_FREEZE_T1);
    const Book& bk = tb.bk[c];  // tables of the round that just ran
    if (!frozen && j < bk.m) {
      const long long num = sb[(c * 16 + j) * 2], den = sb[(c * 16 + j) * 2 + 1];
      if (den > 0) {
        sT[c][bk.idx[j]] = __double2float_rn(__ddiv_rn(__ll2double_rn(num), __ll2double_rn(den)));
        atomicAdd(&s_upd[c], 1);
      }
    }
  }
  __syncthreads();
  const bool f0 = (flags & AAAC_FREEZE_T0) != 0, f1 = (flags & AAAC_FREEZE_T1) != 0;
  const int empty = (f0 ? 0 : n - s_upd[0]) + (f1 ? 0 : n - s_upd[1]);
  build_tables(tb, sT, n, true);
  store_tables(ctl, tb);
  if (tid < 32) {
    const float t = sT[tid >> 4][tid & 15];
    ctl->T[tid >> 4][tid & 15] = t;
    ro.T_user[tid] = t;
  }
  if (tid < 64) (&ctl->bins[0][0][0])[tid] = 0;
  if (tid == 0) {
    // counters other blocks updated with atomics: read them from L2
    ctl->empty_cells = (unsigned long long)empty;
    if (ro.stats) {
      ro.stats->near_ties = (int64_t)__ldcg(&ctl->near_ties);
      ro.stats->groups_t1 = (int64_t)__ldcg(&ctl->groups_t1);
      ro.stats->empty_cells = (int64_t)empty;
      ro.stats->dead_groups = (int64_t)__ldcg(&ctl->dead_groups);
      ro.stats->exact_groups = (int64_t)__ldcg(&ctl->exact_groups);
      ro.stats->L = ctl->L;
      ro.stats->reserved = 0;
    }
    ctl->near_ties = 0;
    ctl->groups_t1 = 0;
    ctl->ticket = 0;
  }
}

template <int FMT, bool PACK>
__global__ void __launch_bounds__(kFitThreads, kFitBlocksPerSM)
fit_pass(const uint16_t* __restrict__ W, int N, int K, const float* __restrict__ I,
         const void* __restrict__ scales, int g, int S, uint32_t flags, FitCtl* ctl,
         double* __restrict__ errp, int ncb, int rows_per_chunk, float tau, PackOut po,
         RoundOut ro) {
  extern __shared__ __align__(16) unsigned char smem[];
  Tables& tb = *reinterpret_cast<Tables*>(smem);
  uint4* ring = reinterpret_cast<uint4*>(smem + ((sizeof(Tables) + 15) & ~(size_t)15));
  ulonglong2* bins = reinterpret_cast<ulonglong2*>(ring + kFitWarps * kStages * 32);
  __shared__ double sred[kFitThreads];
  __shared__ int s_last;

  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&ctl->tb);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&tb);
    for (int i = threadIdx.x; i < (int)(sizeof(Tables) / 4); i += blockDim.x) dst[i] = src[i];
    if (!PACK)
      for (int i = threadIdx.x; i < kFitWarps * 32 * 16; i += blockDim.x)
        bins[i] = make_ulonglong2(0ull, 0ull);
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
  const float la = tb.la;
  uint4* myring = ring + warp * kStages * 32 + lane;
  ulonglong2* mybins = bins + warp * 32 * 16 + (lane >> 1);

  float Ik[8];
  if (active) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(I + col0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(I + col0 + 4));
    Ik[0] = a.x; Ik[1] = a.y; Ik[2] = a.z; Ik[3] = a.w;
    Ik[4] = b.x; Ik[5] = b.y; Ik[6] = b.z; Ik[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++) Ik[i] = 0.0f;
  }

  const int r0 = rc * rows_per_chunk, r1 = min(N, r0 + rows_per_chunk);
  const uint16_t* wcol = W + col0;
  // ring prologue
#pragma unroll
  for (int k = 0; k < kStages; k++) {
    const int rr = r0 + warp + kFitWarps * k;
    if (active && rr < r1) cp_async16(myring + k * 32, wcol + (int64_t)rr * K);
    cp_async_commit();
  }
  // scales prefetched two rows ahead
  float s_next = 0.0f, s_next2 = 0.0f;
  if (active && r0 + warp < r1) s_next = load_scale<FMT>(scales, (int64_t)(r0 + warp) * G + col0 / g);
  if (active && r0 + warp + kFitWarps < r1)
    s_next2 = load_scale<FMT>(scales, (int64_t)(r0 + warp + kFitWarps) * G + col0 / g);

  double err_acc = 0.0;
  unsigned long long n_near = 0, n_exact = 0, n_t1 = 0;
  int slot = 0;
  for (int r = r0 + warp; r < r1; r += kFitWarps) {  // warp-uniform trip count
    cp_async_wait<kStages - 1>();
    const uint4 v = active ? myring[slot * 32] : make_uint4(0, 0, 0, 0);
    const float s = s_next;
    s_next = s_next2;
    if (active && r + 2 * kFitWarps < r1)
      s_next2 = load_scale<FMT>(scales, (int64_t)(r + 2 * kFitWarps) * G + col0 / g);
    float rcp;
    const bool live = active && scale_live(s, &rcp);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float u[8];
    uint32_t mm[8];  // merged cell of each weight
    unsigned long long dd = 0ull;  // (D0, D1) partial sums
    bool crowded = false;
    const unsigned long long rcp2 = f2pack(rcp, rcp);
#pragma unroll
    for (int h = 0; h < 4; h++) {
      const float2 up = f2unpack(f2mul(f2pack(bf16_lo(wv[h]), bf16_hi(wv[h])), rcp2));
      u[2 * h] = live ? up.x : 0.0f;
      u[2 * h + 1] = live ? up.y : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const uint32_t c = tb.mlut[__float_as_uint(bucket_t(u[i], la)) & (kNB - 1)];
      crowded |= (c == kCrowded);
      const uint32_t m = c + (u[i] >= tb.mthr[c] ? 1u : 0u);
      mm[i] = m;
      const unsigned long long vv = *reinterpret_cast<const unsigned long long*>(&tb.mval[m]);
      const unsigned long long e = f2sub(f2pack(u[i], u[i]), vv);
      dd = f2fma(f2pack(Ik[i], Ik[i]), f2mul(e, e), dd);
    }
    if (crowded) {  // rare: a bucket with two or more thresholds; redo the lane exactly
      dd = 0ull;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        int m = 0;
        m += (tb.mthr[m + 15] <= u[i]) ? 16 : 0;
        m += (tb.mthr[m + 7] <= u[i]) ? 8 : 0;
        m += (tb.mthr[m + 3] <= u[i]) ? 4 : 0;
        m += (tb.mthr[m + 1] <= u[i]) ? 2 : 0;
        m += (tb.mthr[m] <= u[i]) ? 1 : 0;
        mm[i] = (uint32_t)m;
        const unsigned long long vv = *reinterpret_cast<const unsigned long long*>(&tb.mval[m]);
        const unsigned long long e = f2sub(f2pack(u[i], u[i]), vv);
        dd = f2fma(f2pack(Ik[i], Ik[i]), f2mul(e, e), dd);
      }
    }
    float d0, d1;
    {
      const float2 dv = f2unpack(dd);
      d0 = dv.x;
      d1 = dv.y;
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
        const double ea = __dsub_rn((double)uj, (double)tb.bk[0].val[book_count(tb.bk[0], uj)]);
        const double eb = __dsub_rn((double)uj, (double)tb.bk[1].val[book_count(tb.bk[1], uj)]);
        E0 = __dadd_rn(E0, __dmul_rn(Ij, __dmul_rn(ea, ea)));
        E1 = __dadd_rn(E1, __dmul_rn(Ij, __dmul_rn(eb, eb)));
      }
      choice = (E1 < E0) ? 1 : 0;
    }
    choice = __shfl_sync(0xffffffffu, choice, leader_lane);

    if (s_leader && live) {
      if (exact) {
        n_exact++;
        if (fabs(E1 - E0) < 1e-6 * fmax(E0, E1)) n_near++;
        if (!PACK) err_acc += (double)(s * s) * (choice ? E1 : E0);  // s*s exact in fp32
      } else {
        if (!single && fabsf(d1 - d0) < 1e-6f * fmaxf(d0, d1)) n_near++;
        if (!PACK) err_acc += (double)(s * s) * (double)(choice ? d1 : d0);
      }
      n_t1 += choice;
    }

    if (!PACK) {
      const double s2L = (double)s * (double)s * twoL;  // exact: s^2 has 16 bits
      const int shift = choice ? 4 : 0;
      ulonglong2* cb_bins = mybins + choice * 16 * 16;
      unsigned long long nums[8], dens[8];
      uint32_t qs[8];
#pragma unroll
      for (int i = 0; i < 8; i++) {
        qs[i] = ((uint32_t)tb.mcell[mm[i]] >> shift) & 15u;
        const double A = __dmul_rn((double)Ik[i], s2L);  // exact: 24 + 16 bits
        nums[i] = (unsigned long long)__double_as_longlong(__fma_rn(A, (double)u[i], kMagic));
        dens[i] = (unsigned long long)__double_as_longlong(__dadd_rn(A, kDenMagic));
      }
      // the two lanes of a pair share bins: update them one lane at a time
#pragma unroll
      for (int half = 0; half < 2; half++) {
        if (live && (lane & 1) == half) {
#pragma unroll
          for (int i = 0; i < 8; i++) {
            ulonglong2 x = cb_bins[qs[i] * 16];
            x.x += nums[i];
            x.y += dens[i];
            cb_bins[qs[i] * 16] = x;
          }
        }
        __syncwarp();
      }
    } else if (active) {
      const Book& bc = tb.bk[choice];
      const int shift = choice ? 4 : 0;
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const uint32_t q = ((uint32_t)tb.mcell[mm[i]] >> shift) & 15u;
        packed |= (uint32_t)bc.idx[q] << (4 * i);
        const float wf = (i & 1) ? bf16_hi(wv[i >> 1]) : bf16_lo(wv[i >> 1]);
        const double wh = (double)s * (double)bc.val[q];
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
    // refill this slot with the row kStages steps ahead
    {
      const int rr = r + kFitWarps * kStages;
      if (active && rr < r1) cp_async16(myring + slot * 32, wcol + (int64_t)rr * K);
      cp_async_commit();
    }
    slot = (slot + 1 == kStages) ? 0 : slot + 1;
  }
  cp_async_wait<0>();

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
  sred[threadIdx.x] = err_acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < kFitThreads; i++) t = __dadd_rn(t, sred[i]);
    errp[blockIdx.x] = t;
  }
  if (!PACK && threadIdx.x < 64) {
    // lane-private raw sums -> exact integers: num is exact modulo 2^51, den
    // modulo 2^52, and every lane's partial is far inside those ranges.
    const int cell = threadIdx.x >> 1, which = threadIdx.x & 1;
    long long sum = 0;
    for (int w = 0; w < kFitWarps; w++) {
      const ulonglong2* p = bins + (w * 32 + cell) * 16;
      for (int l = 0; l < 16; l++) {
        const unsigned long long raw = which ? p[l].y : p[l].x;
        sum += which ? (long long)(raw & ((1ull << 52) - 1))
                     : ((long long)(raw << 13) >> 13);
      }
    }
    if (sum) atomicAdd(reinterpret_cast<unsigned long long*>(&ctl->bins[0][0][0]) + threadIdx.x,
                       (unsigned long long)sum);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&ctl->ticket, 1u) == gridDim.x - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (!PACK) {
    round_finalize(ctl, tb, errp, gridDim.x, flags, ro, sred);
  } else {
    double part = 0.0;
    for (int b = threadIdx.x; b < (int)gridDim.x; b += blockDim.x)
      part = __dadd_rn(part, __ldcg(errp + b));
    __syncthreads();
    sred[threadIdx.x] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
      double e = 0.0;
      for (int i = 0; i < kFitThreads; i++) e = __dadd_rn(e, sred[i]);
      if (po.err_final) *po.err_final = e;
      ctl->ticket = 0;
    }
  }
}

static float choice_tau(int S) {
  int lg = 0;
  while ((8 << lg) < S) lg++;
  return (float)((12 + lg) * ldexp(1.0, -22));
}

template <int FMT, bool PACK>
static cudaError_t set_smem() {
  return cudaFuncSetAttribute(fit_pass<FMT, PACK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_bytes(PACK));
}

template <int FMT>
static cudaError_t launch_fit_t(const uint16_t* W, int64_t N, int64_t K, const float* I,
                                const void* scales, int g, int S, int iters, uint32_t flags,
                                float* T, double* err_hist, aaac_stats* stats, void* ws,
                                cudaStream_t st) {
  // per call: the attribute belongs to the current device's copy of the kernel
  const cudaError_t attr = set_smem<FMT, false>();
  if (attr != cudaSuccess) return attr;
  const PassPlan pp = fit_plan(N, K);
  const PassPlan pprep = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  double* errp = reinterpret_cast<double*>(reinterpret_cast<char*>(ws) + fit_ctl_bytes());
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pprep.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl,
                                                   pprep.ncb, pprep.rows_per_chunk);
  fit_setup<<<1, kFitThreads, 0, st>>>(ctl, T, N * K, ncodes(FMT), stats);
  const float tau = choice_tau(S);
  for (int it = 0; it < iters; it++) {
    fit_pass<FMT, false><<<pp.blocks, kFitThreads, smem_bytes(false), st>>>(
        W, (int)N, (int)K, I, scales, g, S, flags, ctl, errp, pp.ncb, pp.rows_per_chunk, tau,
        PackOut{nullptr, nullptr, nullptr, nullptr}, RoundOut{err_hist, T, stats, it});
  }
  count_launches(2 + iters);
  return cudaSuccess;
}

cudaError_t launch_fit(const uint16_t* W, int64_t N, int64_t K, const float* I,
                       const void* scales, int fmt, int g, int S, int iters, uint32_t flags,
                       float* T, double* err_hist, aaac_stats* stats, void* ws, cudaStream_t st) {
  cudaError_t e = (fmt == kInt4)
                      ? launch_fit_t<kInt4>(W, N, K, I, scales, g, S, iters, flags, T, err_hist,
                                            stats, ws, st)
                      : launch_fit_t<kNvfp4>(W, N, K, I, scales, g, S, iters, flags, T, err_hist,
                                             stats, ws, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// library-owned scratch for aaac_fit_layer_fixed_scratch
// ---------------------------------------------------------------------------
// The fit's scratch (control block + one fp64 per block) in a file-scope device
// array: every GPU that loads the library holds it until the process exits.
// All calls share it, so calls whose work overlaps on the GPU would race.
constexpr size_t kFixedScratchBytes = 256 * 1024;
static __device__ __align__(256) unsigned char g_fit_scratch[kFixedScratchBytes];

size_t fixed_scratch_bytes() { return kFixedScratchBytes; }

// In host code g_fit_scratch names a host-side stand-in, not device memory:
// the device address is looked up with cudaGetSymbolAddress, once per device,
// with that device current, and cached.
cudaError_t fixed_scratch_ptr(void** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fit_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// pack
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kFitThreads)
pack_setup(FitCtl* ctl, const float* T_user, int n, uint16_t* T_bf16) {
  __shared__ Tables tb;
  __shared__ float sT[2][16];
  if (threadIdx.x == 0) {
    ctl->n = n;
    tb.la = bucket_scale(ctl);
  }
  if (threadIdx.x < 32) sT[threadIdx.x >> 4][threadIdx.x & 15] = T_user[threadIdx.x];
  __syncthreads();
  if (threadIdx.x < 2) sort_book(sT[threadIdx.x], n);
  __syncthreads();
  if (threadIdx.x < 32) {
    const int b = threadIdx.x >> 4, j = threadIdx.x & 15;
    const unsigned short h = j < n ? __bfloat16_as_ushort(__float2bfloat16_rn(sT[b][j])) : 0;
    T_bf16[threadIdx.x] = h;
    sT[b][j] = __uint_as_float((uint32_t)h << 16);
  }
  __syncthreads();
  build_tables(tb, sT, n, false);
  store_tables(ctl, tb);
  if (threadIdx.x < 32) ctl->T[threadIdx.x >> 4][threadIdx.x & 15] = sT[threadIdx.x >> 4][threadIdx.x & 15];
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

template <int FMT>
static cudaError_t launch_pack_t(const uint16_t* W, int64_t N, int64_t K, const float* I,
                                 const void* scales, int g, int S, uint32_t flags, const float* T,
                                 uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                                 uint8_t* choice_bits, double* err_final, void* ws,
                                 cudaStream_t st) {
  const cudaError_t attr = set_smem<FMT, true>();
  if (attr != cudaSuccess) return attr;
  const PassPlan pp = fit_plan(N, K);
  const PassPlan pprep = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  double* errp = reinterpret_cast<double*>(reinterpret_cast<char*>(ws) + fit_ctl_bytes());
  uint8_t* cbytes = reinterpret_cast<uint8_t*>(ws) + fit_ws_bytes(N, K);
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pprep.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl,
                                                   pprep.ncb, pprep.rows_per_chunk);
  pack_setup<<<1, kFitThreads, 0, st>>>(ctl, T, ncodes(FMT), T_bf16);
  const float tau = choice_tau(S);
  const PackOut po{codes, scales_tagged, cbytes, err_final};
  fit_pass<FMT, true><<<pp.blocks, kFitThreads, smem_bytes(true), st>>>(
      W, (int)N, (int)K, I, scales, g, S, flags, ctl, errp, pp.ncb, pp.rows_per_chunk, tau, po,
      RoundOut{nullptr, nullptr, nullptr, 0});
  int launches = 3;
  if (S != g) {
    const int KS = (int)(K / S);
    const int64_t total = N * ((KS + 7) / 8);
    pack_bits<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(cbytes, N, KS, choice_bits);
    launches++;
  }
  count_launches(launches);
  return cudaSuccess;
}

cudaError_t launch_pack(const uint16_t* W, int64_t N, int64_t K, const float* I,
                        const void* scales, int fmt, int g, int S, uint32_t flags, const float* T,
                        uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                        uint8_t* choice_bits, double* err_final, void* ws, cudaStream_t st) {
  cudaError_t e = (fmt == kInt4)
                      ? launch_pack_t<kInt4>(W, N, K, I, scales, g, S, flags, T, T_bf16, codes,
                                             scales_tagged, choice_bits, err_final, ws, st)
                      : launch_pack_t<kNvfp4>(W, N, K, I, scales, g, S, flags, T, T_bf16, codes,
                                              scales_tagged, choice_bits, err_final, ws, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace aaac
