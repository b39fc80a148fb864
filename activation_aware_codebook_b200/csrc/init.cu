// init.cu -- per-group absmax scales and the quantile initialisation.
//
// "Technical summary: AAAC", section 1 and section 4 (the 4-bit format fixes
// the per-group scale structure: g=128 INT4, g=16 NVFP4) and section 2, core
// mechanism 4, initialisation (T0 and T1 from evenly spaced quantiles of the
// normalised weights, T1 shifted by half a step).
//
//   radix_pass      one pass over W per 8-bit digit of the IEEE total-order
//                   key of u = fp32_RN(w * fp32_RN(1/s)).  The first pass also
//                   computes the scales (absmax of each group: max of the bf16
//                   magnitude bits, reduced over the group's lanes with warp
//                   shuffles; INT4 s = bf16_RN(fp32_RN(a/7)), NVFP4
//                   s = e4m3_RN_satfinite(a)) and counts the top digit with
//                   lanes of equal digits merged (match.any) into per-warp
//                   counts.  Later passes count only keys whose higher digits
//                   match one of the (at most 32) prefixes still being
//                   resolved, found with one probe of a two-entry-bucket hash
//                   table in shared memory.
//   radix_select    one thread per target rank walks its prefix's histogram
//                   and fixes the next digit (4 passes of 8 bits resolve the
//                   32-bit key exactly, ties included); it also builds the
//                   next pass's prefix hash table.
#include "common.cuh"
#include "internal.h"

namespace aaac {

struct InitCtl {
  int64_t rank[32];
  int64_t resid[32];
  uint32_t prefix[32];
  uint32_t slot_prefix[32];
  int32_t nslots;
  int32_t nranks;
  int32_t n;
  uint32_t hmult;           // multiplier of the prefix hash (0: binary search)
  uint4 htab[256];          // bucket: {prefix, slot, prefix, slot}, empty = ~0
  uint32_t hist[32][256];
};

size_t init_ctl_bytes() { return align256(sizeof(InitCtl)); }

PassPlan plan_pass(int64_t N, int64_t K, int target, int seg_cols) {
  PassPlan p;
  p.ncb = (int)((K + seg_cols - 1) / seg_cols);
  int64_t nrc = target / p.ncb;  // at most `target` blocks: one full wave
  if (nrc > N) nrc = N;
  if (nrc < 1) nrc = 1;
  p.rows_per_chunk = (int)((N + nrc - 1) / nrc);
  p.nrc = (int)((N + p.rows_per_chunk - 1) / p.rows_per_chunk);
  p.blocks = p.ncb * p.nrc;
  return p;
}

// Scale of one group from the max of its bf16 magnitude bits; *stored gets
// the stored bits (bf16 for INT4, E4M3 for NVFP4), the result its value.
template <int FMT>
__device__ __forceinline__ float group_scale(uint32_t mx, uint32_t* stored) {
  const float a = __uint_as_float(mx << 16);
  if (FMT == kInt4) {
    const __nv_bfloat16 s = __float2bfloat16_rn(__fdiv_rn(a, 7.0f));
    *stored = __bfloat16_as_ushort(s);
    return __uint_as_float(*stored << 16);
  } else {
    *stored = (uint32_t)__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3);
    return e4m3_mag(*stored & 0x7fu);
  }
}

struct RankInit {
  int64_t rank[32];
};

__global__ void init_setup(InitCtl* c, RankInit ri, int nranks, int n) {
  for (int i = threadIdx.x; i < 32 * 256; i += blockDim.x) (&c->hist[0][0])[i] = 0u;
  if (threadIdx.x < 32) {
    int i = threadIdx.x;
    c->rank[i] = i < nranks ? ri.rank[i] : 0;
    c->resid[i] = c->rank[i];
    c->prefix[i] = 0u;
    c->slot_prefix[i] = 0u;
  }
  if (threadIdx.x == 0) {
    c->nslots = 1;
    c->nranks = nranks;
    c->n = n;
    c->hmult = 0u;
  }
}

// Slot of a prefix: the bucket's two entries are compared (hash table), or a
// binary search over the sorted prefixes when no hash was found.
__device__ __forceinline__ int prefix_slot(uint32_t pre, const uint4* tab, uint32_t mult,
                                           const uint32_t* sp, int nslots) {
  if (mult) {
    const uint4 e = tab[(pre * mult) >> 24];
    return e.x == pre ? (int)e.y : (e.z == pre ? (int)e.w : -1);
  }
  int lo = 0, hi = nslots;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (sp[mid] < pre) lo = mid + 1; else hi = mid;
  }
  return (lo < nslots && sp[lo] == pre) ? lo : -1;
}

template <int FMT, bool FIRST>
__global__ void __launch_bounds__(kThreads)
radix_pass(const uint16_t* __restrict__ W, int N, int K, int g, void* __restrict__ scales,
           InitCtl* c, int pass, int ncb, int rows_per_chunk) {
  __shared__ uint32_t sh[32][256];  // first pass: per-warp counts; else per-slot counts
  __shared__ uint4 tab[256];
  __shared__ uint32_t sp[32];
  __shared__ int ns;
  __shared__ uint32_t smult;
  for (int i = threadIdx.x; i < 32 * 256; i += blockDim.x) (&sh[0][0])[i] = 0u;
  if (!FIRST) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) tab[i] = c->htab[i];
    if (threadIdx.x < 32) sp[threadIdx.x] = c->slot_prefix[threadIdx.x];
    if (threadIdx.x == 0) {
      ns = c->nslots;
      smult = c->hmult;
    }
  }
  __syncthreads();
  const int nslots = FIRST ? 1 : ns;
  const uint32_t mult = FIRST ? 0u : smult;
  const int shift = 24 - 8 * pass;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = blockIdx.x % ncb, rc = blockIdx.x / ncb;
  const int col0 = cb * kSegCols + lane * 8;
  const bool active = col0 < K;
  const int lanes_g = g >> 3;
  const int G = K / g;
  const int r0 = rc * rows_per_chunk, r1 = min(N, r0 + rows_per_chunk);
  for (int r = r0 + warp; r < r1; r += kWarps) {  // warp-uniform: every lane takes part
    const uint4 v = active ? __ldg(reinterpret_cast<const uint4*>(W + (int64_t)r * K + col0))
                           : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const int64_t gi = (int64_t)r * G + col0 / g;
    float s;
    if (FIRST) {
      uint32_t mx = 0;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        mx = max(mx, w[i] & 0x7fffu);
        mx = max(mx, (w[i] >> 16) & 0x7fffu);
      }
      for (int o = 1; o < lanes_g; o <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      uint32_t stored;
      s = group_scale<FMT>(mx, &stored);
      if (active && (lane & (lanes_g - 1)) == 0) {
        if (FMT == kInt4) reinterpret_cast<unsigned short*>(scales)[gi] = (unsigned short)stored;
        else reinterpret_cast<unsigned char*>(scales)[gi] = (unsigned char)stored;
      }
    } else {
      s = active ? load_scale<FMT>(scales, gi) : 0.0f;
    }
    float rcp;
    const bool live = scale_live(s, &rcp);
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float wf = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
      const float u = live ? __fmul_rn(wf, rcp) : 0.0f;
      const uint32_t key = order_key(u);
      if (FIRST) {
        // lanes holding the same top digit add once (fewer same-address atomics)
        const uint32_t d = active ? (key >> 24) : 0x100u;
        const uint32_t peers = __match_any_sync(0xffffffffu, d);
        if (d < 256u && lane == __ffs(peers) - 1) atomicAdd(&sh[warp][d], (uint32_t)__popc(peers));
      } else {
        const int slot = prefix_slot(key >> (shift + 8), tab, mult, sp, nslots);
        if (active && slot >= 0) atomicAdd(&sh[slot][(key >> shift) & 255u], 1u);
      }
    }
  }
  __syncthreads();
  if (FIRST) {
    for (int d = threadIdx.x; d < 256; d += blockDim.x) {
      uint32_t t = 0;
      for (int w = 0; w < kWarps; w++) t += sh[w][d];
      if (t) atomicAdd(&c->hist[0][d], t);
    }
  } else {
    for (int i = threadIdx.x; i < nslots * 256; i += blockDim.x) {
      const uint32_t v = (&sh[0][0])[i];
      if (v) atomicAdd(&c->hist[0][0] + i, v);
    }
  }
}

// 256 threads: the histograms are read into shared memory once, then one
// thread per target rank walks its prefix's 256 counts there.
__global__ void __launch_bounds__(256) radix_select(InitCtl* c, int pass, float* T) {
  __shared__ uint32_t hist[32][256];
  __shared__ uint32_t sp[32];
  __shared__ uint32_t newp[32];
  __shared__ int ns;
  __shared__ int bcnt[256];
  __shared__ uint32_t smult;
  const int tid = threadIdx.x;
  const int nr = c->nranks;
  if (tid == 0) ns = c->nslots;
  if (tid < 32) sp[tid] = c->slot_prefix[tid];
  __syncthreads();
  const int nslots = ns;
  for (int j = tid; j < nslots * 256; j += blockDim.x) {
    (&hist[0][0])[j] = (&c->hist[0][0])[j];
    (&c->hist[0][0])[j] = 0u;  // ready for the next pass
  }
  __syncthreads();
  if (tid < nr) {
    int slot = 0;
    if (pass > 0)
      for (int s = 0; s < nslots; s++)
        if (sp[s] == c->prefix[tid]) slot = s;
    int64_t want = c->resid[tid], cum = 0;
    int d = 0;
    for (; d < 255; d++) {
      const int64_t h = hist[slot][d];
      if (cum + h > want) break;
      cum += h;
    }
    c->resid[tid] = want - cum;
    c->prefix[tid] = (pass == 0) ? (uint32_t)d : ((c->prefix[tid] << 8) | (uint32_t)d);
    newp[tid] = c->prefix[tid];
  }
  __syncthreads();
  if (tid == 0) {
    // sorted distinct prefixes for the next pass (T0's and T1's ranks
    // interleave, so sort first)
    for (int a = 1; a < nr; a++) {
      const uint32_t v = newp[a];
      int b = a - 1;
      while (b >= 0 && newp[b] > v) { newp[b + 1] = newp[b]; b--; }
      newp[b + 1] = v;
    }
    int m = 0;
    for (int r = 0; r < nr; r++)
      if (m == 0 || sp[m - 1] != newp[r]) sp[m++] = newp[r];
    c->nslots = m;
    // the next pass's prefix hash: bucket (p * mult) >> 24 of 256, two entries
    // each; multipliers are tried until no bucket receives three prefixes
    uint32_t mult = 0u;
    if (pass < 3) {
      for (int att = 0; att < 64 && mult == 0u; att++) {
        const uint32_t mu = (0x9E3779B1u + 0x6A09E667u * (uint32_t)att) | 1u;
        for (int b = 0; b < 256; b++) bcnt[b] = 0;
        bool ok = true;
        for (int i = 0; i < m && ok; i++) ok = ++bcnt[(sp[i] * mu) >> 24] <= 2;
        if (ok) mult = mu;
      }
    }
    smult = mult;
  }
  __syncthreads();
  if (tid < 32) c->slot_prefix[tid] = sp[tid];
  if (pass < 3) {
    const uint32_t mult = smult;
    // bucket tid: its prefixes in slot order, empty entries ~0
    uint4 e = make_uint4(~0u, ~0u, ~0u, ~0u);
    if (mult) {
      int k = 0;
      const int m = c->nslots;
      for (int i = 0; i < m; i++)
        if ((int)((sp[i] * mult) >> 24) == tid) {
          if (k == 0) { e.x = sp[i]; e.y = (uint32_t)i; }
          else { e.z = sp[i]; e.w = (uint32_t)i; }
          k++;
        }
    }
    c->htab[tid] = e;
    if (tid == 0) c->hmult = mult;
  }
  if (pass == 3 && tid < 32) {
    const int n = c->n;
    const int j = tid & 15, b = tid >> 4;
    T[tid] = j < n ? key_to_float(c->prefix[b * n + j]) : 0.0f;
  }
}

cudaError_t launch_init(const uint16_t* W, int64_t N, int64_t K, int fmt, int g, void* scales,
                        float* T, void* ws, cudaStream_t st) {
  const PassPlan pp = plan_pass(N, K);
  InitCtl* c = reinterpret_cast<InitCtl*>(ws);
  const int n = ncodes(fmt);
  const int64_t M = N * K;
  RankInit ri;
  for (int j = 0; j < n; j++) {
    ri.rank[j] = (int64_t)(((__int128)(2 * j + 1) * M) / (2 * n));
    int64_t r1 = (int64_t)(((__int128)(j + 1) * M) / n);
    ri.rank[n + j] = r1 > M - 1 ? M - 1 : r1;
  }
  for (int j = 2 * n; j < 32; j++) ri.rank[j] = 0;
  init_setup<<<1, 256, 0, st>>>(c, ri, 2 * n, n);
  for (int pass = 0; pass < 4; pass++) {
    if (fmt == kInt4) {
      if (pass == 0)
        radix_pass<kInt4, true><<<pp.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, g, scales, c,
                                                                pass, pp.ncb, pp.rows_per_chunk);
      else
        radix_pass<kInt4, false><<<pp.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, g, scales, c,
                                                                 pass, pp.ncb, pp.rows_per_chunk);
    } else {
      if (pass == 0)
        radix_pass<kNvfp4, true><<<pp.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, g, scales, c,
                                                                 pass, pp.ncb, pp.rows_per_chunk);
      else
        radix_pass<kNvfp4, false><<<pp.blocks, kThreads, 0, st>>>(W, (int)N, (int)K, g, scales,
                                                                  c, pass, pp.ncb, pp.rows_per_chunk);
    }
    radix_select<<<1, 256, 0, st>>>(c, pass, T);
  }
  count_launches(9);
  return cudaGetLastError();
}

}  // namespace aaac
