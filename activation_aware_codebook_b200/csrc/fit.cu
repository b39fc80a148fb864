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
// One fit round is ONE launch of fit_round: a streaming pass over W whose last
// block to finish (atomic ticket, no waiting) does the refine, sorts the books,
// rebuilds the tables and records the error.  Per block: 3 warps; a warp covers
// 512 columns of a row, 16 per lane (32 bytes), and walks the rows of its work
// items with a 2-slot ring filled by cp.async.bulk (one lane issues a row's
// 1 KB copy on an mbarrier).  The grid is one wave (4 blocks, 12 warps, per SM,
// bounded by the refine bins' shared memory: 16 KB a warp; the last block's
// table rebuild borrows the idle rings for its scratch).  fit_pass<PACK> is the
// pack's pass (final assign, codes, choice bits, weight-space error) on the
// same work distribution with a cp.async ring; fit_pass<fit> is kept as the
// round of the fixed-scratch entry point, which has no room for the per-fit
// scale pairs fit_round reads.
//
// Nearest entry in both books at once (exact):
//   the midpoint thresholds of both books, merged and deduplicated (at most
//   30), split the u line into merged cells; cell m fixes both books' nearest
//   values mv0[m], mv1[m] and bin offsets moff[m].  bucket b = rint(u * la +
//   64) (one FMA); mlut[b] = the number c of merged thresholds at or below
//   every u of the bucket, then m = c + (u >= mthr[c]) -- exact, because every
//   threshold is the smallest fp32 above an exact midpoint.  A bucket holding
//   two or more thresholds maps to the sentinel cell kCrowded whose values are
//   NaN: the NaN reaches the lane's error sums and the lane redoes its 16
//   weights with a binary search.  Every lookup array is 4 bytes per entry and
//   at most 33 entries long, so each warp-wide lookup is one shared-memory
//   wavefront.
// Choice: fp32 group sums when their gap exceeds the rounding bound, else the
//   sequential fp64 rule (the group's leader lane recomputes it).
// Refine sums: per weight R_k(A 2^L u) and R_k(A 2^L), A = I_k s^2, R_k = floor
//   for even columns k and ceil for odd ones.  Each lane owns 32 bins (book,
//   entry) of (num, den) held as fp64 with biases 1.5 * 2^52 and 2^52, where
//   every value is an integer and the spacing is 1: one FMA / ADD rounded
//   toward -inf (+inf) adds floor (ceil) of the exact term, so every partial
//   sum is exact whatever the order, as long as it stays below 2^51 -- the
//   launch plan bounds the rows per lane to keep it there.  Bins are laid out
//   [book*16 + entry][lane] in 16-byte cells: a warp's read-modify-write of
//   its bins touches 32 distinct bank quads, with no conflicts.
#include <cuda.h>

#include <cstddef>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace aaac {

constexpr int kNB = 128;                  // bucket LUT entries
constexpr int kFitWarps = 3;
constexpr int kFitThreads = kFitWarps * 32;
constexpr int kStages = 2;                // rows per warp in flight
constexpr int kFitBlocksPerSM = 4;
constexpr int kPrepRows = 4;  // rows per lane loaded ahead by fit_prep
constexpr int kLaneCols = 16;             // columns per lane
constexpr int kItemRows = 6;              // rows of one work item
constexpr int kMaxStrips = 256;           // per-strip work counters (more strips: one counter)
constexpr int kWarpCols = 32 * kLaneCols; // columns per warp (one row segment)
constexpr int kRingRowBytes = kWarpCols * 2;
constexpr int kCellBytes = 32 * 16;       // one (book, entry) row of a warp's bins
constexpr int kWarpBinBytes = 32 * kCellBytes;
constexpr float kBucketMagic = 12582912.0f;           // 1.5 * 2^23
constexpr double kNumBias = 6755399441055744.0;       // 1.5 * 2^52
constexpr double kDenBias = 4503599627370496.0;       // 2^52
#define kInf __int_as_float(0x7f800000)

// Merged tables of both books (see the header comment).  Entries past the
// last cell are padding (mthr = +inf); 33 entries keep every lookup in bounds.
constexpr int kMerged = 33;
constexpr uint32_t kCrowded = 31;  // lut value of a crowded bucket (base counts are <= 30)
struct Tables {
  float mthr[kMerged];     // merged thresholds, ascending, +inf padded
  float mv0[kMerged];      // book-0 value of merged cell m (NaN at kCrowded)
  float mv1[kMerged];      // book-1 value of merged cell m (NaN at kCrowded)
  uint32_t moff[kMerged];  // bin offsets of cell m: book 0 low 16 bits, book 1 high
  uint8_t mlut[kNB];       // bucket -> merged base count, kCrowded = crowded bucket
  uint8_t mlut4[kNB];      // 4 * mlut: the base count as a byte offset into the 4-byte arrays
  Book bk[2];
  float la;
  int32_t nm;              // number of merged thresholds
  int32_t pad[2];
};
constexpr int kTablesBytes = (int)((sizeof(Tables) + 127) & ~(size_t)127);

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
  // A round's integer sums, contiguous: a row-sharded fit adds them over the
  // shards with one int64 sum-reduction of kShardSums values.
  long long bins[2][16][2];
  unsigned long long err_acc;  // sum of rint(s^2 D 2^Le) of the running pass
  unsigned long long err_fine;  // the same at 2^30 times the scale (see objective_value)
  unsigned long long near_ties;
  unsigned long long groups_t1;
  unsigned long long exact_groups;
  unsigned long long empty_cells;
  unsigned long long exact_total;   // row-sharded fit: exact decisions of earlier rounds
  unsigned long long shard_max[3];  // row-sharded fit: Imax, Umax, S2max bits (max-reduced)
  unsigned int ticket;
  unsigned int next_item;  // work-item counter of the running pass (many strips)
  unsigned int strip_next[kMaxStrips];  // per-strip item counters of the running pass
  double twoLe;            // fixed-point scale of the objective sums
};
constexpr int kShardSums = 64 + 5;  // bins, err_acc, err_fine, near_ties, groups_t1, exact_groups
static_assert(offsetof(FitCtl, exact_groups) == offsetof(FitCtl, bins) + (kShardSums - 1) * 8,
              "the round sums must be contiguous");

size_t fit_ctl_bytes() { return align256(sizeof(FitCtl)); }

// Scale pairs per row of the pair table: the group count rounded up to even.
__host__ __device__ inline int pair_stride(int G) { return G + (G & 1); }

// Work items: kItemRows rows of one 512-column strip; warps claim them from
// a global counter.  A lane's refine partial over its rows (16 terms a row,
// each below 2^B) must stay below 2^50, which caps the items a warp may
// claim; the grid is one wave, or more when the caps need more warps.
struct FitPlan {
  int ncb, cpc, items, max_items, blocks;
};

// M: the weights of the whole layer (of every row shard), which fixes B.
// Concurrent (AAAC_CONCURRENT): one block per kConcurrentWeights weights of
// this call's rows, at least kConcurrentMinBlocks, for layers that share the
// GPU with other layers' passes (measured on the Llama-3-8B-shaped block, 7
// linears on concurrent streams: 14.12 ms per step with full grids, 13.1 ms).
constexpr int64_t kConcurrentWeights = 196608;
constexpr int64_t kConcurrentMinBlocks = 16;
// bps: blocks per SM of one full wave.
static FitPlan fit_plan(int64_t N, int64_t K, int64_t M, bool concurrent,
                        int bps = kFitBlocksPerSM) {
  FitPlan p;
  p.ncb = (int)((K + kWarpCols - 1) / kWarpCols);
  p.cpc = (int)((N + kItemRows - 1) / kItemRows);
  p.items = p.ncb * p.cpc;
  int c = 0;
  while (((int64_t)1 << c) < M) c++;
  const int Bmax = (61 - c) < 40 ? (61 - c) : 40;
  const int64_t cap_rows = ((int64_t)1 << (50 - Bmax)) / kLaneCols;  // >= 64
  p.max_items = (int)(cap_rows / kItemRows);
  const int64_t per_block = (int64_t)kFitWarps * p.max_items;
  const int64_t need = (p.items + per_block - 1) / per_block;
  const int64_t useful = (p.items + kFitWarps - 1) / kFitWarps;
  int64_t blocks = 148 * (int64_t)bps;
  if (concurrent) {
    int64_t share = (N * K + kConcurrentWeights - 1) / kConcurrentWeights;
    if (share < kConcurrentMinBlocks) share = kConcurrentMinBlocks;
    if (blocks > share) blocks = share;
  }
  if (blocks > useful) blocks = useful;
  if (blocks < need) blocks = need;
  p.blocks = (int)blocks;
  return p;
}

void fit_launch_plan(int64_t N, int64_t K, int64_t M_total, uint32_t flags, int32_t out[5]) {
  const FitPlan p = fit_plan(N, K, M_total, (flags & AAAC_CONCURRENT) != 0);
  out[0] = p.blocks;
  out[1] = p.ncb;
  out[2] = p.cpc;
  out[3] = kItemRows;
  out[4] = p.max_items;
}

// The fit's workspace: the control block (work counters, sums, tables), then
// the (s, 1/s_eff) pair of every scale group.
size_t fit_ws_bytes(int64_t N, int64_t K, int g) {
  return fit_ctl_bytes() + align256((size_t)N * (size_t)pair_stride(K / g) * sizeof(float2));
}

size_t pack_extra_bytes(int64_t N, int64_t K, int S) {
  return align256((size_t)N * (size_t)(K / S));
}

static size_t smem_bytes(bool pack) {
  size_t b = kTablesBytes + (size_t)kFitWarps * kStages * kRingRowBytes;
  if (!pack) b += (size_t)kFitWarps * kWarpBinBytes;
  return b;
}

// Claim counters for a pass of wt warps: warp g first takes chunk g / ncb of
// strip g % ncb without a claim (so it can start before the previous round
// has finished); the counters start past those chunks.
__device__ void seed_claims(FitCtl* ctl, int wt, int cpc, int n_items) {
  const int ncb = n_items / cpc;
  for (int i = threadIdx.x; i < kMaxStrips; i += blockDim.x) {
    unsigned v = 0u;
    if (i < ncb && i < wt) v = (unsigned)min((wt - i + ncb - 1) / ncb, cpc);
    ctl->strip_next[i] = v;
  }
  if (threadIdx.x == 0) ctl->next_item = (unsigned)min(wt, n_items);
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

// All tables from the codebooks sT[2][16] (shared memory), by the threads of
// one block (blockDim >= 64; warp 0 does the per-entry work, lane = book * 16
// + entry):
//   1. sort (optional; stable ranks in IEEE total order), then the distinct
//      values (-0 == +0) by ballot, and their exact midpoint thresholds;
//   2. merge: each threshold takes a unique slot (book 0 before an equal
//      book-1 value), equal neighbours collapse to one merged threshold, and
//      the counts of each book's thresholds at or below it come from prefix
//      masks of the slots' sources;
//   3. merged cells: nearest values and bin offsets of both books; the
//      sentinel cell kCrowded holds NaN;
//   4. bucket table: a histogram of the thresholds' buckets and a warp scan;
//      bucket b counts the thresholds below it or opening it, and is crowded
//      when two or more fall strictly inside.
// When sort_first, sT is left sorted (the callers write it back as T).
// Shared-memory scratch of the table rebuild and the refine.  The fit pass's
// last block places it in its (by then idle) row ring, so the pass holds no
// static shared memory for work that only one block does.
struct FinalizeScratch {
  float s_sorted[2][16];
  float s_slot[32];
  int s_src[32];
  int s_cc[2][kMerged];
  int s_A[kNB + 2], s_F[kNB + 2];
  float sT[2][16];
  long long sb[64];
  int s_upd[2];
};

__device__ void build_tables(Tables& tb, float (*sT)[16], int n, bool sort_first,
                             FinalizeScratch& sc) {
  float (*s_sorted)[16] = sc.s_sorted;
  float* s_slot = sc.s_slot;
  int* s_src = sc.s_src;
  int (*s_cc)[kMerged] = sc.s_cc;
  int* s_A = sc.s_A;
  int* s_F = sc.s_F;
  const int tid = threadIdx.x, lane = tid & 31;
  const unsigned full = 0xffffffffu;
  for (int i = tid; i < kNB + 2; i += blockDim.x) {
    s_A[i] = 0;
    s_F[i] = 0;
  }
  if (tid < 32) {
    const int c = lane >> 4, j = lane & 15;
    // 1. sort and distinct values
    const float v = sT[c][j];
    if (sort_first) {
      const uint32_t kv = order_key(v);
      int rk = 0;
      for (int i = 0; i < n; i++) {
        const uint32_t ki = order_key(sT[c][i]);
        rk += (ki < kv || (ki == kv && i < j)) ? 1 : 0;
      }
      if (j < n) s_sorted[c][rk] = v;
    } else if (j < n) {
      s_sorted[c][j] = v;
    }
    __syncwarp();
    const float w = j < n ? s_sorted[c][j] : 0.0f;
    if (sort_first && j < n) sT[c][j] = w;
    const bool distinct = j < n && (j == 0 || !(w == s_sorted[c][j - 1]));
    const unsigned mine = (__ballot_sync(full, distinct) >> (16 * c)) & 0xffffu;
    const int m = __popc(mine);
    Book& bk = tb.bk[c];
    if (distinct) {
      const int pos = __popc(mine & ((1u << j) - 1u));
      bk.val[pos] = w;
      bk.idx[pos] = j;
    }
    __syncwarp();
    if (j >= m) {
      bk.val[j] = bk.val[m - 1];
      bk.idx[j] = bk.idx[m - 1];
    }
    if (j == 0) bk.m = m;
    __syncwarp();
    bk.thr[j] = (j + 1 < m) ? midpoint_threshold(bk.val[j], bk.val[j + 1]) : kInf;
    __syncwarp();
    // 2. merge
    const int na = tb.bk[0].m - 1, nb = tb.bk[1].m - 1;
    const bool have = (c == 0) ? (j < na) : (j < nb);
    if (have) {
      const float t = bk.thr[j];
      int slot = j;
      if (c == 0) {
        for (int q = 0; q < nb; q++) slot += (tb.bk[1].thr[q] < t) ? 1 : 0;
      } else {
        for (int q = 0; q < na; q++) slot += (tb.bk[0].thr[q] <= t) ? 1 : 0;
      }
      s_slot[slot] = t;
      s_src[slot] = c;
    }
    __syncwarp();
    const int ns = na + nb;  // <= 30
    const bool in = lane < ns;
    const float t = in ? s_slot[lane] : 0.0f;
    const bool keep = in && (lane == 0 || !(t == s_slot[lane - 1]));
    const bool dup_next = in && lane + 1 < ns && t == s_slot[lane + 1];
    const unsigned kb = __ballot_sync(full, keep);
    const unsigned from0 = __ballot_sync(full, in && s_src[lane] == 0);
    const unsigned from1 = __ballot_sync(full, in && s_src[lane] == 1);
    const int nm = __popc(kb);
    if (keep) {
      const int idx = __popc(kb & ((1u << lane) - 1u));
      const int end = lane + (dup_next ? 1 : 0);  // last slot equal to t
      const unsigned upto = (end >= 31) ? full : ((2u << end) - 1u);
      tb.mthr[idx] = t;
      s_cc[0][idx + 1] = __popc(from0 & upto);
      s_cc[1][idx + 1] = __popc(from1 & upto);
    }
    if (lane == 0) {
      tb.nm = nm;
      s_cc[0][0] = 0;
      s_cc[1][0] = 0;
    }
  }
  __syncthreads();
  // 3. cells
  const int nm = tb.nm;
  for (int m = tid; m < kMerged; m += blockDim.x) {
    if (m >= nm) tb.mthr[m] = kInf;
    if (m == (int)kCrowded) {
      tb.mv0[m] = __int_as_float(0x7fc00000);
      tb.mv1[m] = __int_as_float(0x7fc00000);
      tb.moff[m] = 0;
    } else {
      const int c0 = m <= nm ? s_cc[0][m] : 0, c1 = m <= nm ? s_cc[1][m] : 0;
      tb.mv0[m] = tb.bk[0].val[c0];
      tb.mv1[m] = tb.bk[1].val[c1];
      tb.moff[m] = (uint32_t)(c0 * kCellBytes) | ((uint32_t)((16 + c1) * kCellBytes) << 16);
    }
  }
  // 4. bucket table
  if (tid < nm) {
    const float th = tb.mthr[tid];
    const int rb = bucket_raw(th, tb.la);                                  // -1 .. kNB
    const bool first = bucket_raw(nextafterf(th, -kInf), tb.la) < rb;     // th opens its bucket
    atomicAdd(&s_A[rb + 1], 1);
    if (first) atomicAdd(&s_F[rb + 1], 1);
  }
  __syncthreads();
  if (tid < 32) {
    // exclusive prefix P[k] = sum of A[k' < k], 5 entries per lane
    int v[5], sum = 0;
#pragma unroll
    for (int i = 0; i < 5; i++) {
      const int k = lane * 5 + i;
      v[i] = k < kNB + 2 ? s_A[k] : 0;
      sum += v[i];
    }
    int incl = sum;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 5; i++) {
      const int k = lane * 5 + i;  // k = b + 1 for bucket b
      if (k >= 1 && k <= kNB) {
        const int base = run + s_F[k];
        const int inner = v[i] - s_F[k];
        tb.mlut[k - 1] = (uint8_t)(inner > 1 ? kCrowded : base);
        tb.mlut4[k - 1] = (uint8_t)(4 * (inner > 1 ? kCrowded : base));
      }
      run += v[i];
    }
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
// rsc (optional): per (row, scale group) the stored scale's magnitude s and
// r = fp32_RN(1/s_eff) of the effective scale, or (s, 0) for a dead group --
// what every fit round needs of the scales, computed once per fit.  Rows are
// pair_stride(K/g) pairs apart (an even count: 16-byte aligned rows).
template <int FMT>
__global__ void __launch_bounds__(kThreads)
fit_prep(const uint16_t* __restrict__ W, int N, int K, const float* __restrict__ I,
         const void* __restrict__ scales, int g, FitCtl* ctl, int ncb, int rows_per_chunk,
         const float* __restrict__ gsc, float2* __restrict__ rsc) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float gsv = FMT == kNvfp4G ? __ldg(gsc) : 1.0f;
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
    // kPrepRows rows per lane are loaded before any is used (loads in flight)
    for (int rb = r0 + warp; rb < r1; rb += kWarps * kPrepRows) {
      float sv[kPrepRows];
      uint4 wv[kPrepRows];
#pragma unroll
      for (int k = 0; k < kPrepRows; k++) {
        // unconditional loads: a row past the chunk reads the chunk's last
        // row, which is not used
        const int r = rb + k * kWarps;
        const int rr = r < r1 ? r : r1 - 1;
        sv[k] = load_scale<FMT>(scales, (int64_t)rr * G + col0 / g);
        wv[k] = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)rr * K + col0));
      }
#pragma unroll
      for (int k = 0; k < kPrepRows; k++) {
        if (rb + k * kWarps >= r1) break;  // warp-uniform
        const float s = sv[k];
        float rcp;
        const bool live = scale_live(eff_scale<FMT>(s, gsv), &rcp);
        dead += (!live && (lane & (lanes_g - 1)) == 0) ? 1ull : 0ull;
        if (rsc && (lane & (lanes_g - 1)) == 0)
          rsc[(int64_t)(rb + k * kWarps) * pair_stride(G) + col0 / g] = make_float2(s, rcp);
        if (live) s2m = fmax(s2m, (double)s * (double)s);
        const uint32_t w[4] = {wv[k].x, wv[k].y, wv[k].z, wv[k].w};
        uint32_t rm = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
          const float wf = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
          rm = max(rm, __float_as_uint(fabsf(__fmul_rn(wf, rcp))));
        }
        um = max(um, live ? rm : 0u);  // a dead group's weights are not counted
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    im = max(im, __shfl_xor_sync(0xffffffffu, im, o));
    um = max(um, __shfl_xor_sync(0xffffffffu, um, o));
    s2m = fmax(s2m, __shfl_xor_sync(0xffffffffu, s2m, o));
    dead += __shfl_xor_sync(0xffffffffu, dead, o);
  }
  // one atomic per block and quantity (same-address atomics serialise)
  __shared__ uint32_t s_im[kWarps], s_um[kWarps];
  __shared__ double s_s2[kWarps];
  __shared__ unsigned long long s_dead[kWarps];
  if (lane == 0) {
    s_im[warp] = im;
    s_um[warp] = um;
    s_s2[warp] = s2m;
    s_dead[warp] = dead;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kWarps; w++) {
      im = max(im, s_im[w]);
      um = max(um, s_um[w]);
      s2m = fmax(s2m, s_s2[w]);
      dead += s_dead[w];
    }
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

// 2^Le for the objective sums: every contribution is a group's s^2 D (or a
// row's weight-space error), rounded to an integer after scaling by 2^Le.
// Both are below M * I_max * S2_max * g2 * (2 U_max)^2 in total (|u - T| <=
// 2 U_max, |w - s T| <= 2 sqrt(S2_max g2) U_max, g2 the square of a per-tensor
// scale for the weight-space error, else 1), and Le keeps that bound below
// 2^61, so the int64 sums cannot overflow and do not depend on the order of
// addition.
__device__ double objective_scale(const FitCtl* ctl, int64_t M, double g2 = 1.0) {
  const double Imax = (double)__uint_as_float(ctl->Imax_bits);
  const double S2max = __longlong_as_double((long long)ctl->S2max_bits);
  const double Umax = (double)__uint_as_float(ctl->Umax_bits);
  const double bound = (double)M * Imax * S2max * g2 * 4.0 * Umax * Umax;
  if (!(bound > 0.0)) return 1.0;
  int Le = 61 - frexp_exponent(bound);
  if (Le > 1000) Le = 1000;
  if (Le < -1000) Le = -1000;
  return ldexp(1.0, Le);
}

// The objective is summed in fixed point so that its value does not depend on
// the order of the additions.  2^Le comes from a bound on the whole sum that
// is rigorous but loose (every weight at the largest importance, scale and
// error), so one unit can be a sizeable part of a group's contribution: with
// many groups below a unit the rounding biases the total.  A second sum at
// 2^30 times the scale keeps that rounding far below the result; it is the
// one used unless the coarse total shows it may have overflowed (2^31 coarse
// units or more, where the coarse sum is itself fine enough).
constexpr double kFineScale = 1073741824.0;  // 2^30
__device__ __forceinline__ double objective_value(unsigned long long coarse,
                                                  unsigned long long fine, double twoLe) {
  return coarse < (1ull << 31) ? (double)(long long)fine / (twoLe * kFineScale)
                               : (double)(long long)coarse / twoLe;
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

static_assert(sizeof(FinalizeScratch) <= (size_t)kFitWarps * kStages * kRingRowBytes,
              "the last block's finalize scratch lives in the row ring");
static_assert(kFitThreads >= 64, "the bin flush takes one thread per (cell, num | den)");

// L = B - E(I_max) - E(S2_max) - max(0, E(U_max)), B = min(40, 61 - ceil(log2 M))
__global__ void __launch_bounds__(kFitThreads)
fit_setup(FitCtl* ctl, float* T_user, int64_t M, int n, aaac_stats* st, int wt, int cpc,
          int n_items) {
  __shared__ Tables tb;
  __shared__ FinalizeScratch sc;
  seed_claims(ctl, wt, cpc, n_items);
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
    ctl->twoLe = objective_scale(ctl, M);
    ctl->err_acc = 0ull;
    ctl->err_fine = 0ull;
    ctl->n = n;
    tb.la = bucket_scale(ctl);
  }
  float (*sT)[16] = sc.sT;
  if (threadIdx.x < 32) sT[threadIdx.x >> 4][threadIdx.x & 15] = T_user[threadIdx.x];
  __syncthreads();
  build_tables(tb, sT, n, true, sc);
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
__device__ void round_finalize(FitCtl* ctl, Tables& tb, uint32_t flags, const RoundOut& ro,
                               int wt, int cpc, int n_items, double g2, FinalizeScratch& sc) {
  float (*sT)[16] = sc.sT;
  long long* sb = sc.sb;
  int* s_upd = sc.s_upd;
  const int tid = threadIdx.x;
  if (tid < 64) sb[tid] = __ldcg(&ctl->bins[0][0][0] + tid);
  if (tid < 32) sT[tid >> 4][tid & 15] = ctl->T[tid >> 4][tid & 15];
  if (tid < 2) s_upd[tid] = 0;
  if (tid == 0) {
    const double acc = objective_value(__ldcg(&ctl->err_acc), __ldcg(&ctl->err_fine), ctl->twoLe);
    // the rounds sum s^2 D with the stored scale factor; a per-tensor scale
    // enters the objective once, as g2 = gs^2
    if (ro.err_hist) ro.err_hist[ro.it] = __dmul_rn(acc, g2);
    ctl->err_acc = 0ull;
    ctl->err_fine = 0ull;
  }
  __syncthreads();
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
  build_tables(tb, sT, n, true, sc);
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
  seed_claims(ctl, wt, cpc, n_items);
}

// Chunk j (16 bytes) of a warp's 1 KB row segment sits at ring slot j ^ bit 3
// of j: the lanes of a quarter warp then read eight distinct bank quads.
__device__ __forceinline__ int ring_slot(int j) { return j ^ ((j >> 3) & 1); }

// fp32 errors of one pair of weights against both books: dd0 += I (u - v0)^2,
// dd1 += I (u - v1)^2, lane x of each pair the even column, lane y the odd one.
__device__ __forceinline__ void pair_errors(unsigned long long u2, unsigned long long I2,
                                            float v0x, float v0y, float v1x, float v1y,
                                            unsigned long long& dd0, unsigned long long& dd1) {
  const unsigned long long e0 = f2sub(u2, f2pack(v0x, v0y));
  const unsigned long long e1 = f2sub(u2, f2pack(v1x, v1y));
  dd0 = f2fma(I2, f2mul(e0, e0), dd0);
  dd1 = f2fma(I2, f2mul(e1, e1), dd1);
}

// Merged cell of u by binary search over the merged thresholds (crowded buckets).
__device__ __forceinline__ uint32_t merged_search(const Tables& tb, float u) {
  uint32_t m = 0;
  m += (tb.mthr[m + 15] <= u) ? 16 : 0;
  m += (tb.mthr[m + 7] <= u) ? 8 : 0;
  m += (tb.mthr[m + 3] <= u) ? 4 : 0;
  m += (tb.mthr[m + 1] <= u) ? 2 : 0;
  m += (tb.mthr[m] <= u) ? 1 : 0;
  return m;
}

// The sequential fp64 errors of one group (section 2, core mechanism 2; the
// oracle's rule): E_c = sum_j I_j (u_j - T_c[nearest])^2 in column order.
__device__ void exact_group_errors(const uint16_t* __restrict__ wrow, const float* __restrict__ Ig,
                                   int n, float rcp, const Tables& tb, double* E0, double* E1) {
  double a = 0.0, b = 0.0;
  for (int j = 0; j < n; j++) {
    const float wf = __uint_as_float((uint32_t)wrow[j] << 16);
    const float uj = __fmul_rn(wf, rcp);
    const double Ij = (double)Ig[j];
    const double ea = __dsub_rn((double)uj, (double)tb.bk[0].val[book_count(tb.bk[0], uj)]);
    const double eb = __dsub_rn((double)uj, (double)tb.bk[1].val[book_count(tb.bk[1], uj)]);
    a = __dadd_rn(a, __dmul_rn(Ij, __dmul_rn(ea, ea)));
    b = __dadd_rn(b, __dmul_rn(Ij, __dmul_rn(eb, eb)));
  }
  *E0 = a;
  *E1 = b;
}

// fp32 choice when the gap clears the rounding bound; else `exact` is set.
__device__ __forceinline__ int fast_choice(float d0, float d1, float tau, bool* exact) {
  const float sum = __fadd_rn(d0, d1);
  const float gap = fabsf(__fsub_rn(d1, d0));
  const bool decided = (sum >= 8.673617379884035e-19f) && (sum < 3.0e38f) &&
                       (gap > __fmul_rn(tau, sum));
  *exact = !decided;
  return (decided && d1 < d0) ? 1 : 0;
}

struct GroupStats {
  unsigned int near, exact, t1;
  unsigned long long err;   // sum of rint(contribution * 2^Le), modulo 2^64
  unsigned long long errf;  // sum of rint(contribution * 2^Le * 2^30)
};

__device__ __forceinline__ void add_objective(GroupStats& gs, double e, double twoLe) {
  gs.err += (unsigned long long)__double2ll_rn(e * twoLe);
  gs.errf += (unsigned long long)__double2ll_rn(e * (twoLe * kFineScale));
}

// Counters of one live group: near ties, exact decisions, T1 groups, and
// its objective s^2 D in fixed point (scale twoLe).
__device__ __forceinline__ void count_group(GroupStats& gs, bool exact, double E0, double E1,
                                            float d0, float d1, int ch, float s, double twoLe) {
  double e;
  if (exact) {
    gs.exact++;
    if (fabs(E1 - E0) < 1e-6 * fmax(E0, E1)) gs.near++;
    e = (double)(s * s) * (ch ? E1 : E0);  // s*s exact in fp32
  } else {
    // never true for a decided group: its gap exceeds tau (d0 + d1) > 1e-6 max
    if (fabsf(d1 - d0) < 1e-6f * fmaxf(d0, d1)) gs.near++;
    e = (double)(s * s) * (double)(ch ? d1 : d0);
  }
  add_objective(gs, e, twoLe);
  gs.t1 += ch;
}

// SC: the selection group size when it is 8 or 16 (the common layouts,
// compiled with S known), or 0 for S >= 32 taken from S_rt.
template <int FMT, bool PACK, int SC>
__global__ void __launch_bounds__(kFitThreads, kFitBlocksPerSM)
fit_pass(const uint16_t* __restrict__ W, int N, int K, const float* __restrict__ I,
         const void* __restrict__ scales, int g, int S_rt, uint32_t flags, FitCtl* ctl,
         int cpc, int n_items, int max_items, float tau, PackOut po,
         RoundOut ro, const float* __restrict__ gsc, int finalize) {
  const int S = SC ? SC : S_rt;
  extern __shared__ __align__(128) unsigned char smem[];
  Tables& tb = *reinterpret_cast<Tables*>(smem);
  unsigned char* ring = smem + kTablesBytes;
  unsigned char* bins = ring + kFitWarps * kStages * kRingRowBytes;
  __shared__ int s_last;

  // ---- up to the dependency wait nothing is read that the previous round
  // writes (W, I and the scales do not change between rounds), so this part
  // can run while the previous round's last block is still finishing.
  if (!PACK) {
    double2* b = reinterpret_cast<double2*>(bins);
    for (int i = threadIdx.x; i < kFitWarps * kWarpBinBytes / 16; i += blockDim.x)
      b[i] = make_double2(kNumBias, kDenBias);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  const int G = K / g, KS = K / S;
  const int lg = __ffs(g) - 1;              // g is a power of two
  const int lanes_s = S >> 4;               // lanes per choice group when S >= 16
  const int leader_lane = S >= 16 ? (lane & ~(lanes_s - 1)) : lane;
  const bool single = (flags & AAAC_SINGLE_CODEBOOK) != 0;
  const float gsv = FMT == kNvfp4G ? __ldg(gsc) : 1.0f;  // written before the fit starts
  unsigned char* wring = ring + warp * kStages * kRingRowBytes;
  const int wr0 = ring_slot(lane) * 16, wr1 = ring_slot(32 + lane) * 16;
  const int rd0 = ring_slot(2 * lane) * 16, rd1 = ring_slot(2 * lane + 1) * 16;
  unsigned char* mybins = bins + warp * kWarpBinBytes + lane * 16;

  // ---- the warp's rows: work items (kItemRows rows of one 512-column strip)
  // in a small FIFO that the W prefetch fills and the row loop drains.  The
  // first item is fixed (chunk gw / ncb of strip gw % ncb, gw the warp's index
  // in the grid); the rest are claimed from counters, one claim in flight
  // ahead of its use.  Strips: a warp stays on its home strip and moves to the
  // next one when it runs dry (per-strip counters keep the importance
  // registers unchanged); with more than kMaxStrips strips a single counter
  // hands out items in order.
  __shared__ int s_fifo[kFitWarps][8];   // item strip, -1 = no more items
  __shared__ int s_fifoc[kFitWarps][8];  // item chunk within its strip
  int* fifo = s_fifo[warp];
  int* fifoc = s_fifoc[warp];
  const int ncb = n_items / cpc;
  const bool per_strip = ncb <= kMaxStrips;
  const int gw = (int)blockIdx.x * kFitWarps + warp;
  int cur_strip = gw % ncb, tried = 0;
  int first = -1, first_c = 0;  // strip and chunk of the fixed item
  if (per_strip) {
    if (gw / ncb < cpc) {
      first = cur_strip;
      first_c = gw / ncb;
    }
  } else if (gw < n_items) {
    first = gw / cpc;
    first_c = gw - first * cpc;
  }
  unsigned pend = 0u;
  bool pend_ok = false, no_more = first < 0;  // no fixed item: nothing is left
  int claimed = first >= 0 ? 1 : 0, tail = 1;
  if (lane == 0) {
    fifo[0] = first;
    fifoc[0] = first_c;
  }
  __syncwarp();
  auto claim = [&]() {  // warp-uniform: start one claim
    pend_ok = !no_more && claimed < max_items;
    if (pend_ok) {
      if (lane == 0)
        pend = per_strip ? atomicAdd(&ctl->strip_next[cur_strip], 1u) : atomicAdd(&ctl->next_item, 1u);
      claimed++;
    }
  };
  auto land_push = [&]() {  // the pending claim's item (or -1) into the FIFO, next claim
    int it = -1, itc = 0;
    while (pend_ok) {
      const int v = __shfl_sync(full, (int)pend, 0);
      if (!per_strip) {
        if (v < n_items) {
          it = v / cpc;
          itc = v - it * cpc;
        }
        break;
      }
      if (v < cpc) {
        it = cur_strip;
        itc = v;
        break;
      }
      claimed--;  // this strip has run dry: try the next one
      if (++tried >= ncb) break;
      cur_strip = cur_strip + 1 == ncb ? 0 : cur_strip + 1;
      claim();
    }
    if (it < 0) no_more = true;
    if (lane == 0) {
      fifo[tail & 7] = it;
      fifoc[tail & 7] = itc;
    }
    tail++;
    __syncwarp();
    claim();
  };

  // prefetch cursor: FIFO position pq, next row pr and end pe of that item,
  // and the item's strip values (set when the cursor enters the item)
  int pq = 0, pr = 0, pe = 0, pgi = 0;
  const uint16_t* psrc = W;
  bool pc0 = false, pc1 = false, pact = false;
  auto enter = [&](int it, int itc) {
    if (it < 0) return;
    const int pseg = it * kWarpCols;
    pr = itc * kItemRows;
    pe = min(N, pr + kItemRows);
    psrc = W + pseg + lane * 8;
    pc0 = pseg + lane * 8 < K;
    pc1 = pseg + 256 + lane * 8 < K;
    const int pcol0 = pseg + lane * kLaneCols;
    pact = pcol0 < K;
    pgi = pact ? (pcol0 >> lg) : 0;
  };
  // the row at the prefetch cursor into ring slot ps; returns its scale
  auto issue = [&](int ps) -> float {
    const uint16_t* src = psrc + (int64_t)pr * K;
    if (pc0) cp_async16(wring + ps * kRingRowBytes + wr0, src);
    if (pc1) cp_async16(wring + ps * kRingRowBytes + wr1, src + 256);
    return pact ? load_scale<FMT>(scales, (int64_t)pr * G + pgi) : 0.0f;
  };
  auto prefetch = [&](int ps) -> float {
    float sc = 0.0f;
    if (fifo[pq & 7] >= 0) {
      sc = issue(ps);
      if (++pr >= pe) {
        pq++;
        if (pq == tail) land_push();
        enter(fifo[pq & 7], fifoc[pq & 7]);
      }
    }
    cp_async_commit();
    return sc;
  };
  enter(first, first_c);
  // ring prologue, first part: rows of the fixed item that do not end it
  float sqv[kStages];
  int npre = 0;
#pragma unroll
  for (int k = 0; k < kStages; k++) {
    sqv[k] = 0.0f;
    if (first >= 0 && npre == k && pr + 1 < pe) {
      sqv[k] = issue(k);
      pr++;
      cp_async_commit();
      npre++;
    }
  }

  // consumer cursor: FIFO position cq, row cr, item end ce, strip ccb; and
  // the strip whose importance is loaded (the fixed item's, before the wait)
  int cq = 0, cr = 0, ce = 0, ccb = 0;
  auto centre = [&](int it, int itc) {
    if (it < 0) return;
    ccb = it;
    cr = itc * kItemRows;
    ce = min(N, cr + kItemRows);
  };
  centre(first, first_c);
  int cur_cb = -1, col0 = 0;
  bool active = false;
  unsigned long long I2[8];
  double Id[16];
  auto load_importance = [&](int cb) {  // fp32 pairs (choice) and fp64 (refine)
    cur_cb = cb;
    col0 = cb * kWarpCols + lane * kLaneCols;
    active = col0 < K;
    float Iv[16];
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const float4 a = active ? __ldg(reinterpret_cast<const float4*>(I + col0) + q)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      Iv[4 * q] = a.x; Iv[4 * q + 1] = a.y; Iv[4 * q + 2] = a.z; Iv[4 * q + 3] = a.w;
    }
#pragma unroll
    for (int p = 0; p < 8; p++) I2[p] = f2pack(Iv[2 * p], Iv[2 * p + 1]);
#pragma unroll
    for (int i = 0; i < 16; i++) Id[i] = (double)Iv[i];
  };
  if (first >= 0) load_importance(ccb);

  // ---- the previous round's results: tables, fixed-point scales, counters
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&ctl->tb);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&tb);
    for (int i = threadIdx.x; i < (int)(sizeof(Tables) / 4); i += blockDim.x) dst[i] = src[i];
  }
  const double twoL = ctl->twoL;
  const double twoLe = ctl->twoLe;
  __syncthreads();
  const float la = tb.la;
  claim();
  // ring prologue, second part: the remaining positions (may claim)
#pragma unroll
  for (int k = 0; k < kStages; k++)
    if (k >= npre) sqv[k] = prefetch(k);

  GroupStats gs{0u, 0u, 0u, 0ull, 0ull};
  int slot = 0;
  const unsigned long long la2 = f2pack(la, la);
  const unsigned long long cc2 = f2pack(kBucketMagic + (float)(kNB / 2), kBucketMagic + (float)(kNB / 2));
  while (true) {  // warp-uniform
    if (fifo[cq & 7] < 0) break;
    const int r = cr;
    const int cb = ccb;
    if (cb != cur_cb) load_importance(cb);
    if (++cr >= ce) {
      cq++;
      centre(fifo[cq & 7], fifoc[cq & 7]);  // already pushed: the prefetch runs ahead
    }
    cp_async_wait<kStages - 1>();
    __syncwarp();  // the row's chunks were copied by other lanes
    const unsigned char* srow = wring + slot * kRingRowBytes;
    const uint4 va = *reinterpret_cast<const uint4*>(srow + rd0);
    const uint4 vb = *reinterpret_cast<const uint4*>(srow + rd1);
    __syncwarp();  // every lane has read the slot before it is refilled
    const float s = sqv[0];
#pragma unroll
    for (int k = 0; k + 1 < kStages; k++) sqv[k] = sqv[k + 1];
    sqv[kStages - 1] = prefetch(slot);  // the row kStages positions ahead into this slot
    slot = (slot + 1 == kStages) ? 0 : slot + 1;

    float rcp;
    const bool live = active && scale_live(eff_scale<FMT>(s, gsv), &rcp);  // dead: u = +-0
    const uint32_t wv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
    const unsigned long long rr2 = f2pack(rcp, rcp);
    unsigned long long u2[8];
#pragma unroll
    for (int p = 0; p < 8; p++) u2[p] = f2mul(f2pack(bf16_lo(wv[p]), bf16_hi(wv[p])), rr2);

    // nearest entries of both books, and the fp32 group errors
    uint32_t moffs[16];
    unsigned long long dd0[2] = {0ull, 0ull}, dd1[2] = {0ull, 0ull};
#pragma unroll
    for (int p = 0; p < 8; p++) {
      const float2 uf = f2unpack(u2[p]);
      const float2 bf = f2unpack(f2fma(u2[p], la2, cc2));
      const uint32_t cx = tb.mlut[__float_as_uint(bf.x) & (kNB - 1)];
      const uint32_t cy = tb.mlut[__float_as_uint(bf.y) & (kNB - 1)];
      const uint32_t mx = cx + (uf.x >= tb.mthr[cx] ? 1u : 0u);
      const uint32_t my = cy + (uf.y >= tb.mthr[cy] ? 1u : 0u);
      moffs[2 * p] = tb.moff[mx];
      moffs[2 * p + 1] = tb.moff[my];
      pair_errors(u2[p], I2[p], tb.mv0[mx], tb.mv0[my], tb.mv1[mx], tb.mv1[my], dd0[p >> 2],
                  dd1[p >> 2]);
    }
    float D0[2], D1[2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const float2 a = f2unpack(dd0[h]), b = f2unpack(dd1[h]);
      D0[h] = __fadd_rn(a.x, a.y);
      D1[h] = __fadd_rn(b.x, b.y);
    }
    if (active && isnan(__fadd_rn(D0[0], D0[1]))) {
      // a crowded bucket (rare): redo the lane's weights with the binary search
      dd0[0] = dd0[1] = dd1[0] = dd1[1] = 0ull;
#pragma unroll
      for (int p = 0; p < 8; p++) {
        const float2 uf = f2unpack(u2[p]);
        const uint32_t mx = merged_search(tb, uf.x), my = merged_search(tb, uf.y);
        moffs[2 * p] = tb.moff[mx];
        moffs[2 * p + 1] = tb.moff[my];
        pair_errors(u2[p], I2[p], tb.mv0[mx], tb.mv0[my], tb.mv1[mx], tb.mv1[my], dd0[p >> 2],
                    dd1[p >> 2]);
      }
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const float2 a = f2unpack(dd0[h]), b = f2unpack(dd1[h]);
        D0[h] = __fadd_rn(a.x, a.y);
        D1[h] = __fadd_rn(b.x, b.y);
      }
    }

    // The choice (section 2, core mechanism 2): decided in fp32 when the gap
    // exceeds the fp32 error bound, else by the sequential fp64 rule.  S = 8:
    // the lane holds two groups; S >= 16: a group spans S/16 lanes.
    int ch[2] = {0, 0};
    bool ex[2] = {false, false};
    float g0[2] = {D0[0], D0[1]}, g1[2] = {D1[0], D1[1]};
    // SINGLE_CODEBOOK forces T0, but an undecided group still takes the exact
    // rule below, so that its near-tie count is that of the sequential fp64
    // errors, as for the other variants.
    if (S == 8) {
#pragma unroll
      for (int h = 0; h < 2; h++)
        if (live) {
          ch[h] = fast_choice(D0[h], D1[h], tau, &ex[h]);
          if (single) ch[h] = 0;
        }
    } else {
      float d0 = __fadd_rn(D0[0], D0[1]), d1 = __fadd_rn(D1[0], D1[1]);
      for (int o = 1; o < lanes_s; o <<= 1) {
        d0 = __fadd_rn(d0, __shfl_xor_sync(0xffffffffu, d0, o));
        d1 = __fadd_rn(d1, __shfl_xor_sync(0xffffffffu, d1, o));
      }
      g0[0] = g0[1] = d0;
      g1[0] = g1[1] = d1;
      if (live) {
        ch[0] = fast_choice(d0, d1, tau, &ex[0]);
        if (single) ch[0] = 0;
      }
      ch[1] = ch[0];
      ex[1] = ex[0];
    }
    double E0[2] = {0.0, 0.0}, E1[2] = {0.0, 0.0};
    if (__any_sync(0xffffffffu, ex[0] || ex[1])) {
      const uint16_t* wrow = W + (int64_t)r * K + col0;
      if (S == 8) {
#pragma unroll
        for (int h = 0; h < 2; h++)
          if (ex[h]) {
            exact_group_errors(wrow + 8 * h, I + col0 + 8 * h, 8, rcp, tb, &E0[h], &E1[h]);
            ch[h] = (!single && E1[h] < E0[h]) ? 1 : 0;
          }
      } else {
        if (ex[0] && lane == leader_lane) {
          exact_group_errors(wrow, I + col0, S, rcp, tb, &E0[0], &E1[0]);
          ch[0] = (!single && E1[0] < E0[0]) ? 1 : 0;
        }
        ch[0] = __shfl_sync(0xffffffffu, ch[0], leader_lane);
        ch[1] = ch[0];
      }
    }
    if (live) {
      if (S == 8) {
        count_group(gs, ex[0], E0[0], E1[0], g0[0], g1[0], ch[0], s, PACK ? 0.0 : twoLe);
        count_group(gs, ex[1], E0[1], E1[1], g0[1], g1[1], ch[1], s, PACK ? 0.0 : twoLe);
      } else if (lane == leader_lane) {
        count_group(gs, ex[0], E0[0], E1[0], g0[0], g1[0], ch[0], s, PACK ? 0.0 : twoLe);
      }
    }
    const uint32_t sel0 = ch[0] ? 0x4432u : 0x4410u;  // book-1 or book-0 half of moff
    const uint32_t sel1 = ch[1] ? 0x4432u : 0x4410u;

    if (!PACK) {
      if (live) {
        const double s2L = (double)s * (double)s * twoL;  // exact: s^2 has at most 16 bits
#pragma unroll
        for (int i = 0; i < 16; i++) {
          const uint32_t off = __byte_perm(moffs[i], 0u, i < 8 ? sel0 : sel1);
          double2* bp = reinterpret_cast<double2*>(mybins + off);
          const float2 uf = f2unpack(u2[i >> 1]);
          const double ud = (double)((i & 1) ? uf.y : uf.x);
          const double A = __dmul_rn(Id[i], s2L);  // exact: 24 + 16 bits
          double2 b = *bp;
          if (i & 1) {  // odd column: ceil
            b.x = __fma_ru(A, ud, b.x);
            b.y = __dadd_ru(b.y, A);
          } else {      // even column: floor
            b.x = __fma_rd(A, ud, b.x);
            b.y = __dadd_rd(b.y, A);
          }
          *bp = b;
        }
      }
    } else if (active) {
      double err_w = 0.0;  // weight-space error of this row's 16 weights
      unsigned long long packed = 0ull;
#pragma unroll
      for (int i = 0; i < 16; i++) {
        const int h = i >> 3;
        const uint32_t off = __byte_perm(moffs[i], 0u, h ? sel1 : sel0);
        const uint32_t q = (off / kCellBytes) & 15u;
        const Book& bc = tb.bk[ch[h]];
        packed |= (unsigned long long)bc.idx[q] << (4 * i);
        const float wf = (i & 1) ? bf16_hi(wv[i >> 1]) : bf16_lo(wv[i >> 1]);
        const double wh = (double)eff_scale<FMT>(s, gsv) * (double)bc.val[q];
        const double d = __dsub_rn((double)wf, wh);
        err_w = __fma_rn(Id[i], __dmul_rn(d, d), err_w);
      }
      add_objective(gs, err_w, twoLe);
      *reinterpret_cast<unsigned long long*>(po.codes + ((int64_t)r * K + col0) / 2) = packed;
      if ((lane & ((g >> 4) - 1)) == 0) {
        const int64_t gi = (int64_t)r * G + (col0 >> lg);
        const uint32_t tag = (S == g) ? (uint32_t)ch[0] : 0u;
        if (FMT == kInt4) {
          const uint32_t hs = reinterpret_cast<const unsigned short*>(scales)[gi];
          reinterpret_cast<unsigned short*>(po.tagged)[gi] =
              (unsigned short)((hs & 0x7fffu) | (tag << 15));
        } else {
          const uint32_t bs = reinterpret_cast<const unsigned char*>(scales)[gi];
          reinterpret_cast<unsigned char*>(po.tagged)[gi] = (unsigned char)((bs & 0x7fu) | (tag << 7));
        }
      }
      if (S != g) {
        if (S == 8) {
          po.choice_bytes[(int64_t)r * KS + col0 / 8] = (uint8_t)ch[0];
          po.choice_bytes[(int64_t)r * KS + col0 / 8 + 1] = (uint8_t)ch[1];
        } else if (lane == leader_lane) {
          po.choice_bytes[(int64_t)r * KS + (col0 >> (__ffs(S) - 1))] = (uint8_t)ch[0];
        }
      }
    }
  }
  cp_async_wait<0>();
  // the next round may start its blocks (they wait for this grid to finish
  // before reading anything it writes)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  for (int o = 16; o > 0; o >>= 1) {
    gs.near += __shfl_xor_sync(0xffffffffu, gs.near, o);
    gs.exact += __shfl_xor_sync(0xffffffffu, gs.exact, o);
    gs.t1 += __shfl_xor_sync(0xffffffffu, gs.t1, o);
  }
  if (lane == 0) {
    if (gs.near) atomicAdd(&ctl->near_ties, (unsigned long long)gs.near);
    if (gs.exact) atomicAdd(&ctl->exact_groups, (unsigned long long)gs.exact);
    if (gs.t1) atomicAdd(&ctl->groups_t1, (unsigned long long)gs.t1);
  }
  // objective: integer sums, the same whatever the order
  for (int o = 16; o > 0; o >>= 1) {
    gs.err += __shfl_xor_sync(0xffffffffu, gs.err, o);
    gs.errf += __shfl_xor_sync(0xffffffffu, gs.errf, o);
  }
  if (lane == 0 && gs.err) atomicAdd(&ctl->err_acc, gs.err);
  if (lane == 0 && gs.errf) atomicAdd(&ctl->err_fine, gs.errf);
  __syncthreads();  // every lane's bins are complete
  if (!PACK && threadIdx.x < 64) {
    // lane bins -> exact integer partials (bias removed exactly), one
    // (book, entry, num | den) per thread, summed over the block's lanes
    const int bc = threadIdx.x >> 1, which = threadIdx.x & 1;
    const double bias = which ? kDenBias : kNumBias;
    long long sum = 0;
    for (int w = 0; w < kFitWarps; w++) {
      const unsigned char* p = bins + w * kWarpBinBytes + bc * kCellBytes + which * 8;
      for (int j = 0; j < 32; j++) {
        const int l = (j + bc) & 31;  // staggered: fewer bank conflicts
        sum += __double2ll_rn(__dsub_rn(*reinterpret_cast<const double*>(p + l * 16), bias));
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
  const int wt = (int)gridDim.x * kFitWarps;
  if (!finalize) {
    // row-sharded: the sums are reduced over the shards before the round
    // ends (shard_round_end / shard_pack_end); only the claims are reset
    if (threadIdx.x == 0) ctl->ticket = 0;
    seed_claims(ctl, wt, cpc, n_items);
  } else if (!PACK) {
    round_finalize(ctl, tb, flags, ro, wt, cpc, n_items, __dmul_rn((double)gsv, (double)gsv),
                   *reinterpret_cast<FinalizeScratch*>(ring));  // the ring is idle now
  } else {
    if (threadIdx.x == 0) {
      if (po.err_final)
        *po.err_final = objective_value(__ldcg(&ctl->err_acc), __ldcg(&ctl->err_fine), ctl->twoLe);
      ctl->err_acc = 0ull;
      ctl->err_fine = 0ull;
      ctl->ticket = 0;
    }
    seed_claims(ctl, wt, cpc, n_items);
  }
}

// ---------------------------------------------------------------------------
// the fit round
// ---------------------------------------------------------------------------
// fit_round is fit_pass<fit> rebuilt around the same arithmetic with less work
// per weight and per row:
//   - W arrives by cp.async.bulk: one lane issues a 1 KB row segment into a
//     2-slot ring on an mbarrier (the other lanes compute no addresses);
//   - the scales arrive as (s, 1/s_eff) pairs that fit_prep computes once
//     per fit, instead of a correctly rounded reciprocal per row;
//   - every per-lane decision (live group, choice, objective, refine) is a
//     select: the refine of a dead or inactive lane adds exact zeros, so the
//     row has no divergent branch outside the rare crowded-bucket and exact
//     choice paths;
//   - the bucket table holds byte offsets (4 c), so a cell's address needs no
//     multiply.
// The refine sums, the exact choice and the last block's refine are those of
// fit_pass, so the two give the same tables bit for bit.
constexpr int kRStages = 2;                  // ring rows per warp
constexpr uint64_t kRoundWaitNs = 2000000000ull;

__device__ unsigned int g_fit_timeout = 0;
cudaError_t fit_check_flag(unsigned int* out) {
#ifdef AAAC_CHECKS
  return read_check_flag(out);
#else
  *out = 0u;
  return cudaSuccess;
#endif
}

struct __align__(16) RoundRing {
  unsigned char w[kRStages][kWarpCols * 2];
  unsigned long long bar[kRStages];
  int fifo[8];
  int fifoc[8];
};
constexpr size_t kRoundSmem = kFitWarps * (sizeof(RoundRing) + kWarpBinBytes);

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void bar_init(unsigned long long* b) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(b)) : "memory");
}
__device__ __forceinline__ bool bar_test(unsigned long long* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (about 2 s of the global timer); false and the device flag set
// when it runs out.
__device__ __forceinline__ bool bar_wait(unsigned long long* b, uint32_t parity) {
  if (bar_test(b, parity)) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (!bar_test(b, parity)) {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > kRoundWaitNs) {
      atomicExch(&g_fit_timeout, 1u);
      return false;
    }
  }
  return true;
}

// One row segment (bytes: a multiple of 16, both ends 16-byte aligned) into a
// ring slot, issued by the lane for which `on` holds (guard predicates, no
// branch): the barrier's arrival with the byte count, then the copy.
__device__ __forceinline__ void issue_row(bool on, unsigned long long* b, void* dst,
                                          const void* src, uint32_t bytes) {
  asm volatile(
      "{\n .reg .pred p;\n"
      " setp.ne.u32 p, %0, 0;\n"
      " @p fence.proxy.async.shared::cta;\n"
      " @p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %4;\n"
      " @p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%2], [%3], %4, [%1];\n"
      "}\n" ::"r"((uint32_t)on),
      "r"(smem_addr(b)), "r"(smem_addr(dst)), "l"(src), "r"(bytes)
      : "memory");
}

// Merged cells of one lane-row's 16 weights (u as 8 column pairs): the fp32
// errors D0 / D1 of both books over columns 0-7 and 8-15 (the summation
// structure fit_pass uses, so the same rounding bound holds), and the cells'
// bin offsets.
__device__ __forceinline__ void assign_row(const Tables& tb, const float2 (&u2)[8],
                                           const float2 (&Ip)[8], float la, float (&D0)[2],
                                           float (&D1)[2], uint32_t (&moffs)[16]) {
  const unsigned char* mthr_b = reinterpret_cast<const unsigned char*>(tb.mthr);
  const unsigned char* mv0_b = reinterpret_cast<const unsigned char*>(tb.mv0);
  const unsigned char* mv1_b = reinterpret_cast<const unsigned char*>(tb.mv1);
  const unsigned char* moff_b = reinterpret_cast<const unsigned char*>(tb.moff);
  const float cc = kBucketMagic + (float)(kNB / 2);
  const float2 la2 = make_float2(la, la), cc2 = make_float2(cc, cc), neg1 = make_float2(-1.f, -1.f);
  float2 dd0[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 dd1[2] = {dd0[0], dd0[1]};
#pragma unroll
  for (int p = 0; p < 8; p++) {
    const float2 bf = __ffma2_rn(u2[p], la2, cc2);
    const uint32_t cx = tb.mlut4[__float_as_uint(bf.x) & (kNB - 1)];
    const uint32_t cy = tb.mlut4[__float_as_uint(bf.y) & (kNB - 1)];
    AAAC_CHECK(cx < 4u * kMerged - 4u && cy < 4u * kMerged - 4u, 5, cx | (cy << 8));
    const uint32_t mx = cx + (u2[p].x >= *reinterpret_cast<const float*>(mthr_b + cx) ? 4u : 0u);
    const uint32_t my = cy + (u2[p].y >= *reinterpret_cast<const float*>(mthr_b + cy) ? 4u : 0u);
    const float2 v0 = make_float2(*reinterpret_cast<const float*>(mv0_b + mx),
                                  *reinterpret_cast<const float*>(mv0_b + my));
    const float2 v1 = make_float2(*reinterpret_cast<const float*>(mv1_b + mx),
                                  *reinterpret_cast<const float*>(mv1_b + my));
    moffs[2 * p] = *reinterpret_cast<const uint32_t*>(moff_b + mx);
    moffs[2 * p + 1] = *reinterpret_cast<const uint32_t*>(moff_b + my);
    const float2 e0 = __ffma2_rn(v0, neg1, u2[p]);
    const float2 e1 = __ffma2_rn(v1, neg1, u2[p]);
    dd0[p >> 2] = __ffma2_rn(Ip[p], __fmul2_rn(e0, e0), dd0[p >> 2]);
    dd1[p >> 2] = __ffma2_rn(Ip[p], __fmul2_rn(e1, e1), dd1[p >> 2]);
  }
#pragma unroll
  for (int h = 0; h < 2; h++) {
    D0[h] = __fadd_rn(dd0[h].x, dd0[h].y);
    D1[h] = __fadd_rn(dd1[h].x, dd1[h].y);
  }
}

// The same by binary search over the merged thresholds (crowded buckets).
__device__ __forceinline__ void assign_row_search(const Tables& tb, const float2 (&u2)[8],
                                                  const float2 (&Ip)[8], float (&D0)[2],
                                                  float (&D1)[2], uint32_t (&moffs)[16]) {
  float2 dd0[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 dd1[2] = {dd0[0], dd0[1]};
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int p = 0; p < 8; p++) {
    const uint32_t mx = merged_search(tb, u2[p].x), my = merged_search(tb, u2[p].y);
    const float2 v0 = make_float2(tb.mv0[mx], tb.mv0[my]);
    const float2 v1 = make_float2(tb.mv1[mx], tb.mv1[my]);
    moffs[2 * p] = tb.moff[mx];
    moffs[2 * p + 1] = tb.moff[my];
    const float2 e0 = __ffma2_rn(v0, neg1, u2[p]);
    const float2 e1 = __ffma2_rn(v1, neg1, u2[p]);
    dd0[p >> 2] = __ffma2_rn(Ip[p], __fmul2_rn(e0, e0), dd0[p >> 2]);
    dd1[p >> 2] = __ffma2_rn(Ip[p], __fmul2_rn(e1, e1), dd1[p >> 2]);
  }
#pragma unroll
  for (int h = 0; h < 2; h++) {
    D0[h] = __fadd_rn(dd0[h].x, dd0[h].y);
    D1[h] = __fadd_rn(dd1[h].x, dd1[h].y);
  }
}

// The objective of a group decided in fp32 (its d is an fp32 sum already):
// fp32_RN(s^2 d) in fixed point, added only when the group is counted here.
__device__ __forceinline__ void fast_objective(GroupStats& gs, bool on, float s2, float d,
                                               double twoLe) {
  const double e = on ? (double)__fmul_rn(s2, d) : 0.0;
  gs.err += (unsigned long long)__double2ll_rn(e * twoLe);
  gs.errf += (unsigned long long)__double2ll_rn(e * (twoLe * kFineScale));
}

// SC: the selection group size when it is 8 or 16, or 0 for S >= 32 (S_rt).
// finalize 0: the row-sharded fit (the sums are reduced over the shards and
// a separate kernel refines).
template <int FMT, int SC>
__global__ void __launch_bounds__(kFitThreads, kFitBlocksPerSM)
fit_round(const uint16_t* __restrict__ W, int N, int K, const float* __restrict__ I,
          const float2* __restrict__ rsc, int g, int S_rt, uint32_t flags, FitCtl* ctl, int cpc,
          int n_items, int max_items, float tau, RoundOut ro, const float* __restrict__ gsc,
          int finalize) {
  const int S = SC ? SC : S_rt;
  __shared__ Tables tb;
  __shared__ int s_last;
  extern __shared__ __align__(128) unsigned char smem[];
  RoundRing* rings = reinterpret_cast<RoundRing*>(smem);
  unsigned char* bins = smem + kFitWarps * sizeof(RoundRing);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  RoundRing& rg = rings[warp];

  // ---- up to the dependency wait nothing is read that the previous round
  // writes (W, I and the scale pairs are the layer's)
  {
    double2* b = reinterpret_cast<double2*>(bins);
    for (int i = threadIdx.x; i < kFitWarps * kWarpBinBytes / 16; i += blockDim.x)
      b[i] = make_double2(kNumBias, kDenBias);
    // stale ring bytes are finite weights: an inactive lane's garbage times
    // its zero reciprocal must not make a NaN
    uint4* r = reinterpret_cast<uint4*>(rg.w);
    for (int i = lane; i < kRStages * kWarpCols * 2 / 16; i += 32) r[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // before the copies overwrite it
  }
  if (lane < kRStages) bar_init(&rg.bar[lane]);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncwarp();

  const int G = K / g;
  const int lg = __ffs(g) - 1;
  const int lanes_s = S >> 4;
  const int leader_lane = S >= 16 ? (lane & ~(lanes_s - 1)) : lane;
  const bool single = (flags & AAAC_SINGLE_CODEBOOK) != 0;
  const float gsv = FMT == kNvfp4G ? __ldg(gsc) : 1.0f;
  unsigned char* mybins = bins + warp * kWarpBinBytes + lane * 16;

  // ---- work items (as in fit_pass): a fixed first item, then claims
  int* fifo = rg.fifo;
  int* fifoc = rg.fifoc;
  const int ncb = n_items / cpc;
  const bool per_strip = ncb <= kMaxStrips;
  const int gw = (int)blockIdx.x * kFitWarps + warp;
  int cur_strip = gw % ncb, tried = 0;
  int first = -1, first_c = 0;
  if (per_strip) {
    if (gw / ncb < cpc) {
      first = cur_strip;
      first_c = gw / ncb;
    }
  } else if (gw < n_items) {
    first = gw / cpc;
    first_c = gw - first * cpc;
  }
  unsigned pend = 0u;
  bool pend_ok = false, no_more = first < 0;
  int claimed = first >= 0 ? 1 : 0, tail = 1;
  if (lane == 0) {
    fifo[0] = first;
    fifoc[0] = first_c;
  }
  __syncwarp();
  auto claim = [&]() {
    pend_ok = !no_more && claimed < max_items;
    if (pend_ok) {
      if (lane == 0)
        pend = per_strip ? atomicAdd(&ctl->strip_next[cur_strip], 1u) : atomicAdd(&ctl->next_item, 1u);
      claimed++;
    }
  };
  auto land_push = [&]() {
    int it = -1, itc = 0;
    while (pend_ok) {
      const int v = __shfl_sync(full, (int)pend, 0);
      if (!per_strip) {
        if (v < n_items) {
          it = v / cpc;
          itc = v - it * cpc;
        }
        break;
      }
      if (v < cpc) {
        it = cur_strip;
        itc = v;
        break;
      }
      claimed--;
      if (++tried >= ncb) break;
      cur_strip = cur_strip + 1 == ncb ? 0 : cur_strip + 1;
      claim();
    }
    if (it < 0) no_more = true;
    if (lane == 0) {
      fifo[tail & 7] = it;
      fifoc[tail & 7] = itc;
    }
    tail++;
    __syncwarp();
    claim();
  };

  // prefetch cursor: the row's W segment into a slot by a bulk copy, and its
  // scale pair into the L1 cache (the row loads it when it runs: a register
  // holding a load in flight would stall the loop at its first move)
  int pq = 0, pr = 0, pe = 0, pseg = 0, pgi = 0;
  uint32_t pbytes = 0;
  bool pact = false;
  const int Gs = pair_stride(G);
  auto enter = [&](int it, int itc) {
    if (it < 0) return;
    pseg = it * kWarpCols;
    pr = itc * kItemRows;
    pe = min(N, pr + kItemRows);
    pbytes = 2u * (uint32_t)min(kWarpCols, K - pseg);
    const int pcol0 = pseg + lane * kLaneCols;
    pact = pcol0 < K;
    pgi = pact ? (pcol0 >> lg) : 0;
  };
  auto issue = [&](int ps) {
    issue_row(lane == 0, &rg.bar[ps], rg.w[ps], W + (int64_t)pr * K + pseg, pbytes);
    const float2* sp = rsc + (pact ? (int64_t)pr * Gs + pgi : 0);
    asm volatile("prefetch.global.L1 [%0];" ::"l"(sp));
  };
  auto prefetch = [&](int ps) {
    if (fifo[pq & 7] >= 0) {
      issue(ps);
      if (++pr >= pe) {
        pq++;
        if (pq == tail) land_push();
        enter(fifo[pq & 7], fifoc[pq & 7]);
      }
    }
  };
  enter(first, first_c);
  int npre = 0;
#pragma unroll
  for (int k = 0; k < kRStages; k++) {
    if (first >= 0 && npre == k && pr + 1 < pe) {
      issue(k);
      pr++;
      npre++;
    }
  }

  int cq = 0, cr = 0, ce = 0, ccb = 0;
  auto centre = [&](int it, int itc) {
    if (it < 0) return;
    ccb = it;
    cr = itc * kItemRows;
    ce = min(N, cr + kItemRows);
  };
  centre(first, first_c);
  int cur_cb = -1, col0 = 0;
  bool active = false;
  float2 Ip[8];
  double Id[16];
  auto load_importance = [&](int cb) {
    cur_cb = cb;
    col0 = cb * kWarpCols + lane * kLaneCols;
    active = col0 < K;
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const float4 a = active ? __ldg(reinterpret_cast<const float4*>(I + col0) + q)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      Ip[2 * q] = make_float2(a.x, a.y);
      Ip[2 * q + 1] = make_float2(a.z, a.w);
    }
#pragma unroll
    for (int i = 0; i < 16; i++) Id[i] = (double)((i & 1) ? Ip[i >> 1].y : Ip[i >> 1].x);
  };
  if (first >= 0) load_importance(ccb);

  // ---- the previous round's results
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&ctl->tb);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&tb);
    for (int i = threadIdx.x; i < (int)(sizeof(Tables) / 4); i += blockDim.x) dst[i] = src[i];
  }
  const double twoL = ctl->twoL;
  const double twoLe = ctl->twoLe;
  __syncthreads();
  const float la = tb.la;
  claim();
#pragma unroll
  for (int k = 0; k < kRStages; k++)
    if (k >= npre) prefetch(k);

  GroupStats gs{0u, 0u, 0u, 0ull, 0ull};
  int slot = 0;
  uint32_t phase = 0;  // bit k: parity of slot k's next phase
  bool timed_out = false;
  while (!timed_out) {  // warp-uniform
    if (fifo[cq & 7] < 0) break;
    const int r = cr;
    AAAC_CHECK(r >= 0 && r < N, 2, r);
    AAAC_CHECK(ccb >= 0 && ccb < ncb, 3, ccb);
    AAAC_CHECK(tail - cq <= 8, 4, tail - cq);
    if (ccb != cur_cb) load_importance(ccb);
    if (++cr >= ce) {
      cq++;
      centre(fifo[cq & 7], fifoc[cq & 7]);
    }
    timed_out = __any_sync(full, !bar_wait(&rg.bar[slot], (phase >> slot) & 1u));
    phase ^= 1u << slot;
    const uint4 va = *reinterpret_cast<const uint4*>(rg.w[slot] + 32 * lane);       // columns 0-7
    const uint4 vb = *reinterpret_cast<const uint4*>(rg.w[slot] + 32 * lane + 16);  // 8-15
    const float2 sr = __ldg(rsc + (active ? (int64_t)r * Gs + (col0 >> lg) : 0));
    __syncwarp();  // every lane has read the slot before it is refilled
    if (!timed_out) prefetch(slot);
    slot = (slot + 1 == kRStages) ? 0 : slot + 1;
    if (timed_out) break;

    const float s = active ? sr.x : 0.0f, rcp = active ? sr.y : 0.0f;
    const bool live = active && rcp > 0.0f;  // dead groups carry rcp = 0: u = 0
    const uint32_t wv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
    const float2 rr = make_float2(rcp, rcp);
    float2 u2[8];
#pragma unroll
    for (int p = 0; p < 8; p++) u2[p] = __fmul2_rn(make_float2(bf16_lo(wv[p]), bf16_hi(wv[p])), rr);

    float D0[2], D1[2];
    uint32_t moffs[16];
    assign_row(tb, u2, Ip, la, D0, D1, moffs);
    const bool crowded = active && isnan(__fadd_rn(D0[0], D0[1]));
    if (__any_sync(full, crowded)) {
      // a crowded bucket (rare): the lane's weights by binary search
      if (crowded) assign_row_search(tb, u2, Ip, D0, D1, moffs);
    }

    // the choice (section 2, core mechanism 2): fp32 when the gap clears the
    // rounding bound, else the sequential fp64 rule
    int ch[2] = {0, 0};
    bool ex[2] = {false, false};
    float g0[2] = {D0[0], D0[1]}, g1[2] = {D1[0], D1[1]};
    if (S == 8) {
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int c = fast_choice(D0[h], D1[h], tau, &ex[h]);
        ch[h] = (live && !single) ? c : 0;
        ex[h] = live && ex[h];
      }
    } else {
      float d0 = __fadd_rn(D0[0], D0[1]), d1 = __fadd_rn(D1[0], D1[1]);
      for (int o = 1; o < lanes_s; o <<= 1) {
        d0 = __fadd_rn(d0, __shfl_xor_sync(full, d0, o));
        d1 = __fadd_rn(d1, __shfl_xor_sync(full, d1, o));
      }
      g0[0] = g0[1] = d0;
      g1[0] = g1[1] = d1;
      const int c = fast_choice(d0, d1, tau, &ex[0]);
      ch[0] = ch[1] = (live && !single) ? c : 0;
      ex[0] = ex[1] = live && ex[0];
    }
    const float s2 = __fmul_rn(s, s);  // exact: at most 16 significant bits
    if (__any_sync(full, ex[0] || ex[1])) {
      const uint16_t* wrow = W + (int64_t)r * K + col0;
      double E0[2] = {0.0, 0.0}, E1[2] = {0.0, 0.0};
      if (S == 8) {
#pragma unroll
        for (int h = 0; h < 2; h++)
          if (ex[h]) {
            exact_group_errors(wrow + 8 * h, I + col0 + 8 * h, 8, rcp, tb, &E0[h], &E1[h]);
            ch[h] = (!single && E1[h] < E0[h]) ? 1 : 0;
          }
      } else {
        if (ex[0] && lane == leader_lane) {
          exact_group_errors(wrow, I + col0, S, rcp, tb, &E0[0], &E1[0]);
          ch[0] = (!single && E1[0] < E0[0]) ? 1 : 0;
        }
        ch[0] = __shfl_sync(full, ch[0], leader_lane);
        ch[1] = ch[0];
      }
      // the exactly decided groups' counters and objective s^2 E (fp64)
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const bool mine = ex[h] && (S == 8 || (h == 0 && lane == leader_lane));
        if (mine) {
          gs.exact++;
          if (fabs(E1[h] - E0[h]) < 1e-6 * fmax(E0[h], E1[h])) gs.near++;
          add_objective(gs, (double)s2 * (ch[h] ? E1[h] : E0[h]), twoLe);
        }
      }
    }
    // the groups decided in fp32: their objective and T1 counts (branch-free)
    if (S == 8) {
#pragma unroll
      for (int h = 0; h < 2; h++) {
        fast_objective(gs, live && !ex[h], s2, ch[h] ? g1[h] : g0[h], twoLe);
        gs.t1 += live ? ch[h] : 0;
      }
    } else {
      const bool lead = live && lane == leader_lane;
      fast_objective(gs, lead && !ex[0], s2, ch[0] ? g1[0] : g0[0], twoLe);
      gs.t1 += lead ? ch[0] : 0;
    }

    // refine sums (section 2, core mechanism 4): R_k(A 2^L u) and R_k(A 2^L)
    // into the lane's bin of (chosen book, entry); a dead or inactive lane
    // adds exact zeros (A = 0)
    const uint32_t sel0 = ch[0] ? 0x4432u : 0x4410u;
    const uint32_t sel1 = ch[1] ? 0x4432u : 0x4410u;
    const double s2L = live ? (double)s2 * twoL : 0.0;
#pragma unroll
    for (int i = 0; i < 16; i++) {
      const uint32_t off = __byte_perm(moffs[i], 0u, i < 8 ? sel0 : sel1);
      AAAC_CHECK(off < (uint32_t)(32 * kCellBytes) && (off & (kCellBytes - 1)) == 0, 1, off);
      double2* bp = reinterpret_cast<double2*>(mybins + off);
      const double ud = (double)((i & 1) ? u2[i >> 1].y : u2[i >> 1].x);
      const double A = __dmul_rn(Id[i], s2L);  // exact: 24 + 16 bits
      double2 b = *bp;
      if (i & 1) {  // odd column: ceil
        b.x = __fma_ru(A, ud, b.x);
        b.y = __dadd_ru(b.y, A);
      } else {  // even column: floor
        b.x = __fma_rd(A, ud, b.x);
        b.y = __dadd_rd(b.y, A);
      }
      *bp = b;
    }
  }
  // the next round may start its blocks
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // every phase of the ring has been waited on: the barriers are released
  // before the last block reuses their memory
  __syncwarp();
  if (lane < kRStages)
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_addr(&rg.bar[lane])) : "memory");

  for (int o = 16; o > 0; o >>= 1) {
    gs.near += __shfl_xor_sync(full, gs.near, o);
    gs.exact += __shfl_xor_sync(full, gs.exact, o);
    gs.t1 += __shfl_xor_sync(full, gs.t1, o);
  }
  if (lane == 0) {
    if (gs.near) atomicAdd(&ctl->near_ties, (unsigned long long)gs.near);
    if (gs.exact) atomicAdd(&ctl->exact_groups, (unsigned long long)gs.exact);
    if (gs.t1) atomicAdd(&ctl->groups_t1, (unsigned long long)gs.t1);
  }
  for (int o = 16; o > 0; o >>= 1) {
    gs.err += __shfl_xor_sync(full, gs.err, o);
    gs.errf += __shfl_xor_sync(full, gs.errf, o);
  }
  if (lane == 0 && gs.err) atomicAdd(&ctl->err_acc, gs.err);
  if (lane == 0 && gs.errf) atomicAdd(&ctl->err_fine, gs.errf);
  __syncthreads();  // every lane's bins are complete
  if (threadIdx.x < 64) {
    // lane bins -> exact integer partials (bias removed exactly), one
    // (book, entry, num | den) per thread, summed over the block's lanes
    const int bc = threadIdx.x >> 1, which = threadIdx.x & 1;
    const double bias = which ? kDenBias : kNumBias;
    long long sum = 0;
    for (int w = 0; w < kFitWarps; w++) {
      const unsigned char* p = bins + w * kWarpBinBytes + bc * kCellBytes + which * 8;
      for (int j = 0; j < 32; j++) {
        const int l = (j + bc) & 31;  // staggered: fewer bank conflicts
        sum += __double2ll_rn(__dsub_rn(*reinterpret_cast<const double*>(p + l * 16), bias));
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
  const int wt = (int)gridDim.x * kFitWarps;
  static_assert(sizeof(FinalizeScratch) <= kFitWarps * sizeof(RoundRing), "finalize scratch in the rings");
  if (!finalize) {
    if (threadIdx.x == 0) ctl->ticket = 0;
    seed_claims(ctl, wt, cpc, n_items);
  } else {
    round_finalize(ctl, tb, flags, ro, wt, cpc, n_items, __dmul_rn((double)gsv, (double)gsv),
                   *reinterpret_cast<FinalizeScratch*>(rings));  // the rings are idle now
  }
}

// ---------------------------------------------------------------------------
// row-sharded fit: the pieces between the reductions
// ---------------------------------------------------------------------------
// dir 0: the maxima into shard_max (for a max-reduction); dir 1: back.
__global__ void shard_maxima(FitCtl* ctl, int dir) {
  if (threadIdx.x != 0) return;
  if (dir == 0) {
    ctl->shard_max[0] = ctl->Imax_bits;
    ctl->shard_max[1] = ctl->Umax_bits;
    ctl->shard_max[2] = ctl->S2max_bits;
  } else {
    ctl->Imax_bits = (uint32_t)ctl->shard_max[0];
    ctl->Umax_bits = (uint32_t)ctl->shard_max[1];
    ctl->S2max_bits = ctl->shard_max[2];
  }
}

// The end of a round once its sums hold every shard's: the refine of
// round_finalize on the round's tables, with the exact-decision count kept
// as a running total of the reduced per-round counts.
__global__ void __launch_bounds__(kFitThreads)
shard_round_end(FitCtl* ctl, uint32_t flags, RoundOut ro, int wt, int cpc, int n_items,
                const float* __restrict__ gsc, int fmt) {
  __shared__ Tables tb;
  __shared__ FinalizeScratch sc;
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&ctl->tb);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&tb);
    for (int i = threadIdx.x; i < (int)(sizeof(Tables) / 4); i += blockDim.x) dst[i] = src[i];
  }
  if (threadIdx.x == 0) {
    ctl->exact_total += ctl->exact_groups;
    ctl->exact_groups = ctl->exact_total;
  }
  __syncthreads();
  const double gs = fmt == kNvfp4G ? (double)__ldg(gsc) : 1.0;
  round_finalize(ctl, tb, flags, ro, wt, cpc, n_items, __dmul_rn(gs, gs), sc);
  __syncthreads();
  if (threadIdx.x == 0) ctl->exact_groups = 0ull;  // the next round counts its own
}

__global__ void shard_pack_end(FitCtl* ctl, double* err_final) {
  if (threadIdx.x != 0) return;
  if (err_final) *err_final = objective_value(ctl->err_acc, ctl->err_fine, ctl->twoLe);
  ctl->err_acc = 0ull;
  ctl->err_fine = 0ull;
}

static float choice_tau(int S) {
  int lg = 0;
  while ((8 << lg) < S) lg++;
  return (float)((12 + lg) * ldexp(1.0, -22));
}

// The fit pass compiled for this selection group size, with its shared
// memory attribute set (per call: the attribute belongs to the current
// device's copy of the kernel).
using FitPassFn = void (*)(const uint16_t*, int, int, const float*, const void*, int, int,
                           uint32_t, FitCtl*, int, int, int, float, PackOut, RoundOut,
                           const float*, int);
template <int FMT, bool PACK>
static cudaError_t fit_kernel(int S, FitPassFn* out) {
  const FitPassFn k = S == 8 ? fit_pass<FMT, PACK, 8>
                    : S == 16 ? fit_pass<FMT, PACK, 16> : fit_pass<FMT, PACK, 0>;
  *out = k;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_bytes(PACK));
}

using FitRoundFn = void (*)(const uint16_t*, int, int, const float*, const float2*, int, int,
                            uint32_t, FitCtl*, int, int, int, float, RoundOut, const float*, int);
template <int FMT>
static cudaError_t round_kernel(int S, FitRoundFn* out) {
  const FitRoundFn k = S == 8 ? fit_round<FMT, 8> : S == 16 ? fit_round<FMT, 16> : fit_round<FMT, 0>;
  *out = k;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRoundSmem);
}

// The fit on fit_round: rsc (N * K/g pairs of the caller's workspace) holds
// the scale pairs fit_prep writes.
template <int FMT>
static cudaError_t launch_fit_round_t(const uint16_t* W, int64_t N, int64_t K, const float* I,
                                      const void* scales, int g, int S, int iters, uint32_t flags,
                                      float* T, double* err_hist, aaac_stats* stats, void* ws,
                                      float2* rsc, const float* gsc, cudaStream_t st) {
  FitRoundFn kern;
  const cudaError_t attr = round_kernel<FMT>(S, &kern);
  if (attr != cudaSuccess) return attr;
  const FitPlan pp = fit_plan(N, K, N * K, (flags & AAAC_CONCURRENT) != 0);
  const PassPlan pprep = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pprep.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl,
                                                   pprep.ncb, pprep.rows_per_chunk, gsc, rsc);
  fit_setup<<<1, kFitThreads, 0, st>>>(ctl, T, N * K, ncodes(FMT), stats, pp.blocks * kFitWarps,
                                       pp.cpc, pp.items);
  const float tau = choice_tau(S);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)pp.blocks);
  lc.blockDim = dim3(kFitThreads);
  lc.dynamicSmemBytes = kRoundSmem;
  lc.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  for (int it = 0; it < iters; it++) {
    const cudaError_t e = cudaLaunchKernelEx(&lc, kern, W, (int)N, (int)K, I,
                                             (const float2*)rsc, g, S, flags, ctl, pp.cpc,
                                             pp.items, pp.max_items, tau,
                                             RoundOut{err_hist, T, stats, it}, gsc, 1);
    if (e != cudaSuccess) return e;
  }
  count_launches(2 + iters);
  return cudaSuccess;
}

template <int FMT>
static cudaError_t launch_fit_t(const uint16_t* W, int64_t N, int64_t K, const float* I,
                                const void* scales, int g, int S, int iters, uint32_t flags,
                                float* T, double* err_hist, aaac_stats* stats, void* ws,
                                const float* gsc, cudaStream_t st) {
  // per call: the attribute belongs to the current device's copy of the kernel
  FitPassFn kern;
  const cudaError_t attr = fit_kernel<FMT, false>(S, &kern);
  if (attr != cudaSuccess) return attr;
  const FitPlan pp = fit_plan(N, K, N * K, (flags & AAAC_CONCURRENT) != 0);
  const PassPlan pprep = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pprep.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl,
                                                   pprep.ncb, pprep.rows_per_chunk, gsc, nullptr);
  fit_setup<<<1, kFitThreads, 0, st>>>(ctl, T, N * K, ncodes(FMT), stats, pp.blocks * kFitWarps,
                                       pp.cpc, pp.items);
  const float tau = choice_tau(S);
  // rounds launched with programmatic stream serialization: a round's blocks
  // may start (and prefetch) while the previous launch finishes; they wait
  // with griddepcontrol.wait before reading what it writes
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)pp.blocks);
  lc.blockDim = dim3(kFitThreads);
  lc.dynamicSmemBytes = smem_bytes(false);
  lc.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  for (int it = 0; it < iters; it++) {
    const cudaError_t e = cudaLaunchKernelEx(
        &lc, kern, W, (int)N, (int)K, I, scales, g, S, flags, ctl, pp.cpc, pp.items,
        pp.max_items, tau, PackOut{nullptr, nullptr, nullptr, nullptr},
        RoundOut{err_hist, T, stats, it}, gsc, 1);
    if (e != cudaSuccess) return e;
  }
  count_launches(2 + iters);
  return cudaSuccess;
}

cudaError_t launch_fit(const uint16_t* W, int64_t N, int64_t K, const float* I,
                       const void* scales, int fmt, int g, int S, int iters, uint32_t flags,
                       float* T, double* err_hist, aaac_stats* stats, void* ws, float2* rsc,
                       const float* gsc, cudaStream_t st) {
  if (rsc) {
    const cudaError_t e =
        (fmt == kInt4) ? launch_fit_round_t<kInt4>(W, N, K, I, scales, g, S, iters, flags, T,
                                                   err_hist, stats, ws, rsc, gsc, st)
        : (fmt == kNvfp4) ? launch_fit_round_t<kNvfp4>(W, N, K, I, scales, g, S, iters, flags, T,
                                                       err_hist, stats, ws, rsc, gsc, st)
                          : launch_fit_round_t<kNvfp4G>(W, N, K, I, scales, g, S, iters, flags,
                                                        T, err_hist, stats, ws, rsc, gsc, st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  cudaError_t e =
      (fmt == kInt4) ? launch_fit_t<kInt4>(W, N, K, I, scales, g, S, iters, flags, T, err_hist,
                                           stats, ws, gsc, st)
      : (fmt == kNvfp4) ? launch_fit_t<kNvfp4>(W, N, K, I, scales, g, S, iters, flags, T, err_hist,
                                               stats, ws, gsc, st)
                        : launch_fit_t<kNvfp4G>(W, N, K, I, scales, g, S, iters, flags, T,
                                                err_hist, stats, ws, gsc, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Row-sharded fit: this process fits rows [its N] of a layer of M_total
// weights.  The maxima that fix L, Le and the bucket scale are max-reduced
// over the shards before the first round; each round's integer sums (bins,
// objective, counters) are sum-reduced before its refine, which every shard
// then runs on identical sums -- so every shard holds the same tables, and
// they equal the unsharded fit's bit for bit (the sums are exact integers).
template <int FMT>
static cudaError_t launch_fit_sharded_t(const uint16_t* W, int64_t N, int64_t K, int64_t M_total,
                                        const float* I, const void* scales, int g, int S,
                                        int iters, uint32_t flags, float* T, double* err_hist,
                                        aaac_stats* stats, void* ws, const float* gsc,
                                        Reducer& red, cudaStream_t st) {
  FitRoundFn kern;
  const cudaError_t attr = round_kernel<FMT>(S, &kern);
  if (attr != cudaSuccess) return attr;
  float2* rsc = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(ws) + fit_ctl_bytes());
  const FitPlan pp = fit_plan(N, K, M_total, (flags & AAAC_CONCURRENT) != 0);
  const PassPlan pprep = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pprep.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl,
                                                   pprep.ncb, pprep.rows_per_chunk, gsc, rsc);
  shard_maxima<<<1, 32, 0, st>>>(ctl, 0);
  int launches = 3;
  if (!red.run(ctl->shard_max, 3, AAAC_REDUCE_MAX_I64, st)) return cudaGetLastError();
  if (!red.run(&ctl->dead_groups, 1, AAAC_REDUCE_SUM_I64, st)) return cudaGetLastError();
  shard_maxima<<<1, 32, 0, st>>>(ctl, 1);
  fit_setup<<<1, kFitThreads, 0, st>>>(ctl, T, M_total, ncodes(FMT), stats,
                                       pp.blocks * kFitWarps, pp.cpc, pp.items);
  launches += 2;
  const float tau = choice_tau(S);
  for (int it = 0; it < iters; it++) {
    kern<<<pp.blocks, kFitThreads, kRoundSmem, st>>>(
        W, (int)N, (int)K, I, (const float2*)rsc, g, S, flags, ctl, pp.cpc, pp.items,
        pp.max_items, tau, RoundOut{nullptr, nullptr, nullptr, it}, gsc, 0);
    if (!red.run(&ctl->bins[0][0][0], kShardSums, AAAC_REDUCE_SUM_I64, st)) break;
    shard_round_end<<<1, kFitThreads, 0, st>>>(ctl, flags, RoundOut{err_hist, T, stats, it},
                                               pp.blocks * kFitWarps, pp.cpc, pp.items, gsc, FMT);
    launches += 2;
  }
  count_launches(launches);
  return cudaGetLastError();
}

cudaError_t launch_fit_sharded(const uint16_t* W, int64_t N, int64_t K, int64_t M_total,
                               const float* I, const void* scales, int fmt, int g, int S,
                               int iters, uint32_t flags, float* T, double* err_hist,
                               aaac_stats* stats, void* ws, const float* gsc, Reducer& red,
                               cudaStream_t st) {
  if (fmt == kInt4)
    return launch_fit_sharded_t<kInt4>(W, N, K, M_total, I, scales, g, S, iters, flags, T,
                                       err_hist, stats, ws, gsc, red, st);
  if (fmt == kNvfp4)
    return launch_fit_sharded_t<kNvfp4>(W, N, K, M_total, I, scales, g, S, iters, flags, T,
                                        err_hist, stats, ws, gsc, red, st);
  return launch_fit_sharded_t<kNvfp4G>(W, N, K, M_total, I, scales, g, S, iters, flags, T,
                                       err_hist, stats, ws, gsc, red, st);
}

// ---------------------------------------------------------------------------
// library-owned scratch for aaac_fit_layer_fixed_scratch
// ---------------------------------------------------------------------------
// The fit's scratch (its control block) in a file-scope device array: every
// GPU that loads the library holds it until the process exits.  All calls
// share it, so calls whose work overlaps on the GPU would race.
constexpr size_t kFixedScratchBytes = 256 * 1024;
static __device__ __align__(256) unsigned char g_fit_scratch[kFixedScratchBytes];
static_assert(sizeof(FitCtl) + 255 <= kFixedScratchBytes,
              "the fit's control block must fit the library-owned scratch");

size_t fixed_scratch_bytes() { return kFixedScratchBytes; }

// In host code g_fit_scratch names a host-side stand-in, not device memory:
// the device address is looked up with cudaGetSymbolAddress with the device
// current.  The address belongs to the copy of the module loaded in the
// current context, so it is cached per device together with that context's
// unique id, and looked up again when the current context is another one
// (for example the primary context made anew after cudaDeviceReset).
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
static CtxGetIdFn ctx_get_id_fn() {
  static CtxGetIdFn fn = []() -> CtxGetIdFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetIdFn>(p);
  }();
  return fn;
}

cudaError_t fixed_scratch_ptr(void** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_id[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const CtxGetIdFn get_id = ctx_get_id_fn();
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long id = 0;
  // a NULL context means "the current one"; no id (no context yet, or no
  // driver entry point) means no cached address is trusted
  const bool have_id = get_id && get_id(nullptr, &id) == CUDA_SUCCESS && id != 0;
  if (addr[dev] != nullptr && have_id && ctx_id[dev] == id) {
    *out = addr[dev];
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_fit_scratch);  // makes the device's context current
  if (e != cudaSuccess) return e;
  if (get_id && get_id(nullptr, &id) == CUDA_SUCCESS && id != 0) {
    addr[dev] = p;
    ctx_id[dev] = id;
  } else {
    addr[dev] = nullptr;
  }
  *out = p;
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// pack
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kFitThreads)
pack_setup(FitCtl* ctl, const float* T_user, int64_t M, int n, uint16_t* T_bf16, int wt,
           int cpc, int n_items, const float* gsc) {
  __shared__ Tables tb;
  __shared__ FinalizeScratch sc;
  float (*sT)[16] = sc.sT;
  seed_claims(ctl, wt, cpc, n_items);
  if (threadIdx.x == 0) {
    ctl->n = n;
    const double gs = gsc ? (double)*gsc : 1.0;  // the pack's error is in weight space
    ctl->twoLe = objective_scale(ctl, M, gs * gs);
    ctl->err_acc = 0ull;
    ctl->err_fine = 0ull;
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
  build_tables(tb, sT, n, false, sc);
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
                                 const float* gsc, cudaStream_t st) {
  FitPassFn kern;
  const cudaError_t attr = fit_kernel<FMT, true>(S, &kern);
  if (attr != cudaSuccess) return attr;
  const FitPlan pp = fit_plan(N, K, N * K, (flags & AAAC_CONCURRENT) != 0);
  const PassPlan pprep = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  uint8_t* cbytes = reinterpret_cast<uint8_t*>(ws) + fit_ctl_bytes();
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pprep.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl,
                                                   pprep.ncb, pprep.rows_per_chunk, gsc, nullptr);
  pack_setup<<<1, kFitThreads, 0, st>>>(ctl, T, N * K, ncodes(FMT), T_bf16,
                                        pp.blocks * kFitWarps, pp.cpc, pp.items,
                                        FMT == kNvfp4G ? gsc : nullptr);
  const float tau = choice_tau(S);
  const PackOut po{codes, scales_tagged, cbytes, err_final};
  kern<<<pp.blocks, kFitThreads, smem_bytes(true), st>>>(
      W, (int)N, (int)K, I, scales, g, S, flags, ctl, pp.cpc, pp.items, pp.max_items, tau, po,
      RoundOut{nullptr, nullptr, nullptr, 0}, gsc, 1);
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

// Row-sharded pack: every shard packs its rows with the final tables; the
// fixed-point scale of the error comes from the max-reduced maxima and the
// error is the sum-reduced integer total, as in the unsharded pack.
template <int FMT>
static cudaError_t launch_pack_sharded_t(const uint16_t* W, int64_t N, int64_t K,
                                         int64_t M_total, const float* I, const void* scales,
                                         int g, int S, uint32_t flags, const float* T,
                                         uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                                         uint8_t* choice_bits, double* err_final, void* ws,
                                         const float* gsc, Reducer& red, cudaStream_t st) {
  FitPassFn kern;
  const cudaError_t attr = fit_kernel<FMT, true>(S, &kern);
  if (attr != cudaSuccess) return attr;
  const FitPlan pp = fit_plan(N, K, M_total, (flags & AAAC_CONCURRENT) != 0);
  const PassPlan pprep = plan_pass(N, K);
  FitCtl* ctl = reinterpret_cast<FitCtl*>(ws);
  uint8_t* cbytes = reinterpret_cast<uint8_t*>(ws) + fit_ctl_bytes();
  cudaMemsetAsync(ctl, 0, sizeof(FitCtl), st);
  fit_prep<FMT><<<pprep.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, I, scales, g, ctl,
                                                   pprep.ncb, pprep.rows_per_chunk, gsc, nullptr);
  shard_maxima<<<1, 32, 0, st>>>(ctl, 0);
  int launches = 2;
  if (red.run(ctl->shard_max, 3, AAAC_REDUCE_MAX_I64, st)) {
    shard_maxima<<<1, 32, 0, st>>>(ctl, 1);
    pack_setup<<<1, kFitThreads, 0, st>>>(ctl, T, M_total, ncodes(FMT), T_bf16,
                                          pp.blocks * kFitWarps, pp.cpc, pp.items,
                                          FMT == kNvfp4G ? gsc : nullptr);
    const PackOut po{codes, scales_tagged, cbytes, err_final};
    kern<<<pp.blocks, kFitThreads, smem_bytes(true), st>>>(
        W, (int)N, (int)K, I, scales, g, S, flags, ctl, pp.cpc, pp.items, pp.max_items,
        choice_tau(S), po, RoundOut{nullptr, nullptr, nullptr, 0}, gsc, 0);
    launches += 3;
    if (S != g) {
      const int KS = (int)(K / S);
      const int64_t total = N * ((KS + 7) / 8);
      pack_bits<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(cbytes, N, KS, choice_bits);
      launches++;
    }
    if (red.run(&ctl->err_acc, 2, AAAC_REDUCE_SUM_I64, st)) {  // err_acc, err_fine
      shard_pack_end<<<1, 32, 0, st>>>(ctl, err_final);
      launches++;
    }
  }
  count_launches(launches);
  return cudaGetLastError();
}

cudaError_t launch_pack_sharded(const uint16_t* W, int64_t N, int64_t K, int64_t M_total,
                                const float* I, const void* scales, int fmt, int g, int S,
                                uint32_t flags, const float* T, uint16_t* T_bf16, uint8_t* codes,
                                void* scales_tagged, uint8_t* choice_bits, double* err_final,
                                void* ws, const float* gsc, Reducer& red, cudaStream_t st) {
  if (fmt == kInt4)
    return launch_pack_sharded_t<kInt4>(W, N, K, M_total, I, scales, g, S, flags, T, T_bf16,
                                        codes, scales_tagged, choice_bits, err_final, ws, gsc,
                                        red, st);
  if (fmt == kNvfp4)
    return launch_pack_sharded_t<kNvfp4>(W, N, K, M_total, I, scales, g, S, flags, T, T_bf16,
                                         codes, scales_tagged, choice_bits, err_final, ws, gsc,
                                         red, st);
  return launch_pack_sharded_t<kNvfp4G>(W, N, K, M_total, I, scales, g, S, flags, T, T_bf16,
                                        codes, scales_tagged, choice_bits, err_final, ws, gsc,
                                        red, st);
}

cudaError_t launch_pack(const uint16_t* W, int64_t N, int64_t K, const float* I,
                        const void* scales, int fmt, int g, int S, uint32_t flags, const float* T,
                        uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                        uint8_t* choice_bits, double* err_final, void* ws, const float* gsc,
                        cudaStream_t st) {
  cudaError_t e =
      (fmt == kInt4) ? launch_pack_t<kInt4>(W, N, K, I, scales, g, S, flags, T, T_bf16, codes,
                                            scales_tagged, choice_bits, err_final, ws, gsc, st)
      : (fmt == kNvfp4) ? launch_pack_t<kNvfp4>(W, N, K, I, scales, g, S, flags, T, T_bf16, codes,
                                                scales_tagged, choice_bits, err_final, ws, gsc, st)
                        : launch_pack_t<kNvfp4G>(W, N, K, I, scales, g, S, flags, T, T_bf16,
                                                 codes, scales_tagged, choice_bits, err_final, ws,
                                                 gsc, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace aaac
