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
//   tensor_amax     (NVFP4 with a per-tensor scale only) the largest |w| of
//                   the tensor, as the max of the bf16 magnitude bits; every
//                   radix pass then forms gs = fp32_RN(amax / 448) from it and
//                   the first radix_select stores gs for the caller.
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
  uint32_t amax_bits;       // bf16 magnitude bits of the tensor's largest |w|
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
// With a per-tensor scale gs the stored E4M3 factor is that of a / gs (0 when
// gs is 0: the whole tensor is zero).
template <int FMT>
__device__ __forceinline__ float group_scale(uint32_t mx, uint32_t* stored, float gs) {
  const float a = __uint_as_float(mx << 16);
  if (FMT == kInt4) {
    const __nv_bfloat16 s = __float2bfloat16_rn(__fdiv_rn(a, 7.0f));
    *stored = __bfloat16_as_ushort(s);
    return __uint_as_float(*stored << 16);
  } else if (FMT == kNvfp4) {
    *stored = (uint32_t)__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3);
    return e4m3_mag(*stored & 0x7fu);
  } else {
    *stored = gs > 0.0f ? (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(a, gs), __NV_SATFINITE,
                                                          __NV_E4M3)
                        : 0u;
    return e4m3_mag(*stored & 0x7fu);
  }
}

// gs = fp32_RN(amax / 448), 0 for a zero tensor.
__device__ __forceinline__ float tensor_scale(uint32_t amax_bits) {
  const float a = __uint_as_float(amax_bits << 16);
  return a > 0.0f ? __fdiv_rn(a, 448.0f) : 0.0f;
}

__global__ void __launch_bounds__(kThreads)
tensor_amax(const uint4* __restrict__ W, uint32_t n_vec, InitCtl* c) {
  uint32_t mx = 0;
  for (uint32_t i = blockIdx.x * kThreads + threadIdx.x; i < n_vec; i += gridDim.x * kThreads) {
    const uint4 v = __ldg(W + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; k++) mx = max(mx, max(w[k] & 0x7fffu, (w[k] >> 16) & 0x7fffu));
  }
  for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0 && mx) atomicMax(&c->amax_bits, mx);
}

constexpr int kRadixRows = 4;  // rows per lane loaded ahead in a radix pass

// *p += v in shared memory when cond holds: one predicated reduction, no
// branch (lanes that do not count skip the access).
__device__ __forceinline__ void shared_add_if(uint32_t* p, uint32_t v, bool cond) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q red.shared.add.u32 [%0], %1;\n\t}"
      ::"r"(a), "r"(v), "r"((uint32_t)cond)
      : "memory");
}

// The same at a 32-bit shared address base + 4 idx (idx need not be valid
// where cond is false: the access is then not made).
__device__ __forceinline__ void shared_add_at(uint32_t base, uint32_t idx, uint32_t v, bool cond) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q red.shared.add.u32 [%0], %1;\n\t}"
      ::"r"(base + 4u * idx), "r"(v), "r"((uint32_t)cond)
      : "memory");
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
    c->amax_bits = 0u;
  }
}

struct RadixArgs {
  const uint16_t* W;
  int N, K, g;
  void* scales;
  int pass, ncb, rows_per_chunk;
};

// The rows of one warp.  MODE 0: the first pass (scales, top digit); 1: later
// passes with the prefix hash; 2: later passes with the binary search.
template <int FMT, int MODE>
__device__ __forceinline__ void radix_rows(const RadixArgs& a, uint32_t (*sh)[256], const uint4* tab,
                                           uint32_t mult, const uint32_t* sp, int nslots,
                                           float gs) {
  const int shift = 24 - 8 * a.pass;
  const int K = a.K, g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = blockIdx.x % a.ncb, rc = blockIdx.x / a.ncb;
  const int col0 = cb * kSegCols + lane * 8;
  const bool active = col0 < K;
  const int lanes_g = g >> 3;
  const int G = K / g;
  const int r0 = rc * a.rows_per_chunk, r1 = min(a.N, r0 + a.rows_per_chunk);
  if (MODE != 0 && !active) return;  // no warp collectives in later passes
  const uint32_t sh_base = (uint32_t)__cvta_generic_to_shared(&sh[0][0]);
  const int cl = active ? col0 : K - 8;  // the column a lane loads from
  // kRadixRows rows per lane are loaded before any is processed (loads in flight)
  for (int rb = r0 + warp; rb < r1; rb += kWarps * kRadixRows) {  // warp-uniform
    uint4 vr[kRadixRows];
    float sr[kRadixRows];
#pragma unroll
    for (int k = 0; k < kRadixRows; k++) {
      // unconditional loads: a row past the chunk reads the chunk's last row
      // and a lane past K the last 8 columns; neither value is counted
      const int r = rb + k * kWarps;
      const int rr = r < r1 ? r : r1 - 1;
      vr[k] = __ldg(reinterpret_cast<const uint4*>(a.W + (int64_t)rr * K + cl));
      sr[k] = MODE != 0 ? load_scale<FMT>(a.scales, (int64_t)rr * G + cl / g) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < kRadixRows; k++) {
      const int r = rb + k * kWarps;
      if (r >= r1) break;  // warp-uniform
      const uint32_t w[4] = {vr[k].x, vr[k].y, vr[k].z, vr[k].w};
      float s = sr[k];
      if (MODE == 0) {
        uint32_t mx = 0;
#pragma unroll
        for (int i = 0; i < 4; i++) {
          mx = max(mx, w[i] & 0x7fffu);
          mx = max(mx, (w[i] >> 16) & 0x7fffu);
        }
        for (int o = 1; o < lanes_g; o <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        uint32_t stored;
        s = group_scale<FMT>(mx, &stored, gs);
        if (active && (lane & (lanes_g - 1)) == 0) {
          const int64_t gi = (int64_t)r * G + col0 / g;
          if (FMT == kInt4) reinterpret_cast<unsigned short*>(a.scales)[gi] = (unsigned short)stored;
          else reinterpret_cast<unsigned char*>(a.scales)[gi] = (unsigned char)stored;
        }
      }
      float rcp;
      const bool live = scale_live(eff_scale<FMT>(s, gs), &rcp);
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const float wf = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
        const float u = live ? __fmul_rn(wf, rcp) : 0.0f;
        const uint32_t key = order_key(u);
        if (MODE == 0) {
          // lanes holding the same top digit add once (fewer same-address atomics)
          const uint32_t d = active ? (key >> 24) : 0x100u;
          const uint32_t peers = __match_any_sync(0xffffffffu, d);
          shared_add_if(&sh[warp][d & 255u], (uint32_t)__popc(peers),
                        d < 256u && lane == __ffs(peers) - 1);
        } else {
          const uint32_t pre = key >> (shift + 8);
          uint32_t slot;
          bool hit;
          if (MODE == 1) {  // selects, no branches: slot is only used on a hit
            const uint4 e = tab[(pre * mult) >> 24];
            const bool hx = e.x == pre;
            hit = hx || e.z == pre;
            slot = hx ? e.y : e.w;
          } else {
            int lo = 0, hi = nslots;  // sorted distinct prefixes
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              if (sp[mid] < pre) lo = mid + 1; else hi = mid;
            }
            hit = lo < nslots && sp[lo] == pre;
            slot = (uint32_t)lo;
          }
          AAAC_CHECK(!hit || slot < (uint32_t)nslots, 6, slot);
          shared_add_at(sh_base, slot * 256u + ((key >> shift) & 255u), 1u, hit);
        }
      }
    }
  }
}

template <int FMT, bool FIRST>
__global__ void __launch_bounds__(kThreads)
radix_pass(RadixArgs a, InitCtl* c) {
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
  const float gs = FMT == kNvfp4G ? tensor_scale(c->amax_bits) : 1.0f;
  if (FIRST) radix_rows<FMT, 0>(a, sh, tab, 0u, sp, 1, gs);
  else if (smult) radix_rows<FMT, 1>(a, sh, tab, smult, sp, nslots, gs);
  else radix_rows<FMT, 2>(a, sh, tab, 0u, sp, nslots, gs);
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

// 256 threads.  The histograms are read into shared memory; warp w resolves
// target ranks w, w + 8, ...: a warp scan over its prefix's 256 counts finds
// the digit.  Warp 0 then sorts and deduplicates the new prefixes and builds
// the next pass's prefix hash table (bucket (p * mult) >> 24 of 256, two
// entries each; multipliers are tried until no bucket receives three).
__global__ void __launch_bounds__(256) radix_select(InitCtl* c, int pass, float* T,
                                                    float* gs_out) {
  __shared__ uint32_t hist[32][256];
  __shared__ uint32_t sp[32];
  __shared__ uint32_t newp[32];
  __shared__ uint32_t sorted[32];
  __shared__ uint4 stab[256];
  __shared__ int ns;
  __shared__ uint32_t smult;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned full = 0xffffffffu;
  const int nr = c->nranks;
  if (tid == 0) ns = c->nslots;
  if (tid < 32) sp[tid] = c->slot_prefix[tid];
  __syncthreads();
  const int nslots = ns;
  const int nh = nslots * 256;
  uint32_t* gh = &c->hist[0][0];
  for (int j0 = 0; j0 < nh; j0 += 256 * 8) {  // 8 loads in flight per thread
    uint32_t v[8];
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const int j = j0 + k * 256 + tid;
      v[k] = j < nh ? __ldcg(gh + j) : 0u;
    }
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const int j = j0 + k * 256 + tid;
      if (j < nh) (&hist[0][0])[j] = v[k];
    }
  }
  for (int j = tid; j < nh; j += 256) gh[j] = 0u;  // ready for the next pass (own entries)
  __syncthreads();

  for (int t = warp; t < nr; t += 8) {  // warp-uniform
    int slot = 0;
    const uint32_t pre = c->prefix[t];
    if (pass > 0) {
      const unsigned m = __ballot_sync(full, lane < nslots && sp[lane] == pre);
      slot = m ? __ffs(m) - 1 : 0;
    }
    const int64_t want = c->resid[t];
    uint32_t h[8];
    int64_t loc = 0;
#pragma unroll
    for (int k = 0; k < 8; k++) {
      h[k] = hist[slot][lane * 8 + k];
      loc += h[k];
    }
    int64_t incl = loc;
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += y;
    }
    // first digit d < 255 with (count below d) + h[d] > want, else 255
    int64_t cum = incl - loc, cd = 0;
    int dl = 256;
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const int d = lane * 8 + k;
      if (dl == 256 && d < 255 && cum + (int64_t)h[k] > want) {
        dl = d;
        cd = cum;
      }
      cum += h[k];
    }
    const unsigned hit = __ballot_sync(full, dl < 256);
    int d;
    int64_t below;
    if (hit) {
      const int src = __ffs(hit) - 1;
      d = __shfl_sync(full, dl, src);
      below = __shfl_sync(full, cd, src);
    } else {
      d = 255;
      below = __shfl_sync(full, incl, 31) - (int64_t)__shfl_sync(full, h[7], 31);
    }
    if (lane == 0) {
      c->resid[t] = want - below;
      const uint32_t p = (pass == 0) ? (uint32_t)d : ((pre << 8) | (uint32_t)d);
      c->prefix[t] = p;
      newp[t] = p;
    }
  }
  __syncthreads();

  if (warp == 0) {
    // sorted distinct prefixes (T0's and T1's ranks interleave): stable rank
    const uint32_t v = lane < nr ? newp[lane] : 0xffffffffu;
    int rk = 0;
    for (int j = 0; j < nr; j++) {
      const uint32_t x = __shfl_sync(full, v, j);
      rk += (x < v || (x == v && j < lane)) ? 1 : 0;
    }
    if (lane < nr) sorted[rk] = v;
    __syncwarp();
    const uint32_t sv = lane < nr ? sorted[lane] : 0u;
    const uint32_t prev = __shfl_up_sync(full, sv, 1);
    const bool first = lane < nr && (lane == 0 || prev != sv);
    const unsigned fm = __ballot_sync(full, first);
    const int m = __popc(fm);
    if (first) sp[__popc(fm & ((1u << lane) - 1u))] = sv;
    __syncwarp();
    uint32_t mult = 0u;
    if (pass < 3) {
      for (int att = 0; att < 64; att++) {
        const uint32_t mu = (0x9E3779B1u + 0x6A09E667u * (uint32_t)att) | 1u;
        const uint32_t bk = lane < m ? (sp[lane] * mu) >> 24 : 0x100u + (uint32_t)lane;
        const uint32_t peers = __match_any_sync(full, bk);
        if (__all_sync(full, __popc(peers) <= 2)) {
          mult = mu;
          break;
        }
      }
    }
    if (lane == 0) {
      c->nslots = m;
      smult = mult;
    }
  }
  stab[tid] = make_uint4(~0u, ~0u, ~0u, ~0u);
  __syncthreads();
  const uint32_t mult = smult;
  if (warp == 0 && pass < 3 && mult) {
    const int m = c->nslots;
    const uint32_t bk = lane < m ? (sp[lane] * mult) >> 24 : 0x100u + (uint32_t)lane;
    const uint32_t peers = __match_any_sync(full, bk);
    if (lane < m) {
      if (__popc(peers & ((1u << lane) - 1u)) == 0) {
        stab[bk].x = sp[lane];
        stab[bk].y = (uint32_t)lane;
      } else {
        stab[bk].z = sp[lane];
        stab[bk].w = (uint32_t)lane;
      }
    }
  }
  __syncthreads();
  if (tid < 32) c->slot_prefix[tid] = sp[tid];
  if (pass < 3) {
    c->htab[tid] = stab[tid];
    if (tid == 0) c->hmult = mult;
  }
  if (pass == 0 && gs_out && tid == 0) *gs_out = tensor_scale(c->amax_bits);
  if (pass == 3 && tid < 32) {
    const int n = c->n;
    const int j = tid & 15, b = tid >> 4;
    T[tid] = j < n ? key_to_float(c->prefix[b * n + j]) : 0.0f;
  }
}

template <int FMT>
static void radix_pass_launch(int pass, int blocks, const RadixArgs& a, InitCtl* c,
                              cudaStream_t st) {
  if (pass == 0) radix_pass<FMT, true><<<blocks, kThreads, 0, st>>>(a, c);
  else radix_pass<FMT, false><<<blocks, kThreads, 0, st>>>(a, c);
}

cudaError_t init_check_flag(unsigned int* out) {
#ifdef AAAC_CHECKS
  return read_check_flag(out);
#else
  *out = 0u;
  return cudaSuccess;
#endif
}

cudaError_t launch_init(const uint16_t* W, int64_t N, int64_t K, int fmt, int g, void* scales,
                        float* T, void* ws, float* gs_out, cudaStream_t st) {
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
  int launches = 9;
  if (fmt == kNvfp4G) {
    const uint32_t n_vec = (uint32_t)(M / 8);
    int blocks = (int)((n_vec + kThreads - 1) / kThreads);
    if (blocks > 148 * 8) blocks = 148 * 8;
    tensor_amax<<<blocks, kThreads, 0, st>>>(reinterpret_cast<const uint4*>(W), n_vec, c);
    launches++;
  }
  for (int pass = 0; pass < 4; pass++) {
    const RadixArgs a{W, (int)N, (int)K, g, scales, pass, pp.ncb, pp.rows_per_chunk};
    if (fmt == kInt4) radix_pass_launch<kInt4>(pass, pp.blocks, a, c, st);
    else if (fmt == kNvfp4) radix_pass_launch<kNvfp4>(pass, pp.blocks, a, c, st);
    else radix_pass_launch<kNvfp4G>(pass, pp.blocks, a, c, st);
    radix_select<<<1, 256, 0, st>>>(c, pass, T, fmt == kNvfp4G ? gs_out : nullptr);
  }
  count_launches(launches);
  return cudaGetLastError();
}

// Row-sharded init: this process holds N rows of a layer of M_total weights.
// The target ranks come from M_total; the tensor maximum (NVFP4 with a
// tensor scale) is max-reduced and each pass's histograms are sum-reduced
// over the shards before the select, so every shard selects the same keys:
// the order statistics of the whole layer.
cudaError_t launch_init_sharded(const uint16_t* W, int64_t N, int64_t K, int64_t M_total, int fmt,
                                int g, void* scales, float* T, void* ws, float* gs_out,
                                Reducer& red, cudaStream_t st) {
  const PassPlan pp = plan_pass(N, K);
  InitCtl* c = reinterpret_cast<InitCtl*>(ws);
  const int n = ncodes(fmt);
  const int64_t M = M_total;
  RankInit ri;
  for (int j = 0; j < n; j++) {
    ri.rank[j] = (int64_t)(((__int128)(2 * j + 1) * M) / (2 * n));
    int64_t r1 = (int64_t)(((__int128)(j + 1) * M) / n);
    ri.rank[n + j] = r1 > M - 1 ? M - 1 : r1;
  }
  for (int j = 2 * n; j < 32; j++) ri.rank[j] = 0;
  init_setup<<<1, 256, 0, st>>>(c, ri, 2 * n, n);
  int launches = 1;
  if (fmt == kNvfp4G) {
    const uint32_t n_vec = (uint32_t)(N * K / 8);
    int blocks = (int)((n_vec + kThreads - 1) / kThreads);
    if (blocks > 148 * 8) blocks = 148 * 8;
    tensor_amax<<<blocks, kThreads, 0, st>>>(reinterpret_cast<const uint4*>(W), n_vec, c);
    launches++;
    if (!red.run(&c->amax_bits, 1, AAAC_REDUCE_MAX_I32, st)) {
      count_launches(launches);
      return cudaGetLastError();
    }
  }
  for (int pass = 0; pass < 4; pass++) {
    const RadixArgs a{W, (int)N, (int)K, g, scales, pass, pp.ncb, pp.rows_per_chunk};
    if (fmt == kInt4) radix_pass_launch<kInt4>(pass, pp.blocks, a, c, st);
    else if (fmt == kNvfp4) radix_pass_launch<kNvfp4>(pass, pp.blocks, a, c, st);
    else radix_pass_launch<kNvfp4G>(pass, pp.blocks, a, c, st);
    launches++;
    if (!red.run(&c->hist[0][0], 32 * 256, AAAC_REDUCE_SUM_I32, st)) break;
    radix_select<<<1, 256, 0, st>>>(c, pass, T, fmt == kNvfp4G ? gs_out : nullptr);
    launches++;
  }
  count_launches(launches);
  return cudaGetLastError();
}

}  // namespace aaac
