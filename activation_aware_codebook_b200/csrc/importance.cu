// importance.cu -- column importance I_k = sum_t X[t,k]^2.
//
// "Technical summary: AAAC", section 2, core mechanism 2: each weight column
// is weighted by the activation energy of its input channel over the
// calibration set.  The result is the exact sum rounded once to fp32.
//
// Kernels
//   importance_partial  streams X once with 128-bit coalesced loads: a warp
//                       reads 512 contiguous bytes of a row (32 lanes x 8
//                       columns); each lane keeps 8 fp64 accumulators.  The
//                       square of a bf16 is exact in fp64; the bf16 -> fp64
//                       widening is done with integer ops.  The 8 warps of a
//                       block are combined in a fixed order.
//   importance_finalize one thread per column sums the row-block partials in
//                       fixed order, bounds the rounding error of the whole
//                       fp64 summation tree, and writes fp32_RN(sum) when the
//                       bound decides the rounding; otherwise it queues the
//                       column for the exact path.
//   importance_exact    exact integer sum for queued columns: squares grouped
//                       by bf16 exponent in 64-bit bins (x^2 = M^2 * 4^(e-134)),
//                       then one base-4 carry pass and a round-to-nearest-even.
#include "common.cuh"
#include "internal.h"

namespace aaac {

ImportancePlan plan_importance(int64_t T, int64_t K) {
  ImportancePlan p;
  p.ncb = (int)((K + kSegCols - 1) / kSegCols);
  int target = 148 * 8;
  int64_t rb = (target + p.ncb - 1) / p.ncb;
  int64_t max_rb = (T + kWarps - 1) / kWarps;
  if (rb > max_rb) rb = max_rb;
  if (rb < 1) rb = 1;
  p.rb = (int)rb;
  p.rows_per_rb = (T + rb - 1) / rb;
  p.partial_bytes = align256((size_t)rb * (size_t)K * sizeof(double));
  p.list_bytes = align256((size_t)(K + 1) * sizeof(int32_t));
  p.total = p.partial_bytes + p.list_bytes;
  return p;
}

// |x| of a bf16 widened to fp64 by bit manipulation (exact for normal
// numbers; zeros and subnormals come out below 2^-126, whose squares the
// error bound covers as an absolute slack).
__device__ __forceinline__ double bf16_abs_to_f64(uint32_t h16) {
  return __hiloint2double((int)(((h16 & 0x7fffu) << 13) + 0x38000000u), 0);
}

__global__ void __launch_bounds__(kThreads)
importance_partial(const uint16_t* __restrict__ X, int64_t T, int64_t K, int64_t ldx,
                   int64_t rows_per_rb, double* __restrict__ partial) {
  __shared__ double red[kWarps][kSegCols];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t col0 = (int64_t)blockIdx.x * kSegCols + lane * 8;
  const bool active = col0 < K;
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; i++) acc[i] = 0.0;
  const int64_t t0 = (int64_t)blockIdx.y * rows_per_rb;
  const int64_t t1 = min(T, t0 + rows_per_rb);
  if (active) {
    const uint16_t* p = X + col0;
    for (int64_t t = t0 + warp; t < t1; t += kWarps) {
      uint4 v = __ldg(reinterpret_cast<const uint4*>(p + t * ldx));
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; i++) {
        double a = bf16_abs_to_f64(w[i] & 0xffffu);
        double b = bf16_abs_to_f64(w[i] >> 16);
        acc[2 * i] = __fma_rn(a, a, acc[2 * i]);
        acc[2 * i + 1] = __fma_rn(b, b, acc[2 * i + 1]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; i++) red[warp][lane * 8 + i] = acc[i];
  __syncthreads();
  const int c = threadIdx.x;  // kThreads == kSegCols
  double s = red[0][c];
#pragma unroll
  for (int w = 1; w < kWarps; w++) s = __dadd_rn(s, red[w][c]);
  const int64_t col = (int64_t)blockIdx.x * kSegCols + c;
  if (col < K) partial[(int64_t)blockIdx.y * K + col] = s;
}

__global__ void importance_finalize(const double* __restrict__ partial, int rb, int64_t K,
                                    int accumulate, float* I, double gam, double slack,
                                    int force_exact, int32_t* list, int32_t* nlist) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double s = accumulate ? (double)I[k] : 0.0;
  for (int b = 0; b < rb; b++) s = __dadd_rn(s, partial[(int64_t)b * K + k]);
  const double E = __dadd_ru(__dmul_ru(s, gam), slack);
  const float lo = __double2float_rn(__dsub_rd(s, E));
  const float hi = __double2float_rn(__dadd_ru(s, E));
  if (!force_exact && __float_as_uint(lo) == __float_as_uint(hi)) {
    I[k] = lo;
  } else {
    int at = atomicAdd(nlist, 1);
    list[at] = (int32_t)k;
  }
}

// Round sum_b bins[b] * 4^(b-134) to fp32 (nearest, ties to even).  Binary
// position p carries 2^(p-268); fp32's subnormal quantum 2^-149 is p = 119.
__device__ float exact_bins_to_f32(const unsigned long long* bins) {
  unsigned char dig[320];
  unsigned long long c = 0;
  int nd = 0;
  for (int b = 0; b < 256; b++) {
    c += bins[b];
    dig[nd++] = (unsigned char)(c & 3u);
    c >>= 2;
  }
  while (c && nd < 320) {
    dig[nd++] = (unsigned char)(c & 3u);
    c >>= 2;
  }
  int hb = nd - 1;
  while (hb >= 0 && dig[hb] == 0) hb--;
  if (hb < 0) return 0.0f;
  const int h = 2 * hb + (dig[hb] >> 1);
  const int lo = max(h - 23, 119);
  uint32_t mant = 0;
  for (int p = h; p >= lo; p--) mant = (mant << 1) | ((dig[p >> 1] >> (p & 1)) & 1u);
  const int round = (dig[(lo - 1) >> 1] >> ((lo - 1) & 1)) & 1;
  int sticky = 0;
  for (int p = lo - 2; p >= 0 && !sticky; p--) sticky = (dig[p >> 1] >> (p & 1)) & 1;
  if (round && (sticky || (mant & 1u))) mant++;
  return __double2float_rn(ldexp((double)mant, lo - 268));
}

__global__ void __launch_bounds__(kThreads)
importance_exact(const uint16_t* __restrict__ X, int64_t T, int64_t ldx, int accumulate, float* I,
                 const int32_t* __restrict__ list, const int32_t* __restrict__ nlist) {
  __shared__ unsigned long long bins[256];
  const int n = *nlist;
  for (int li = blockIdx.x; li < n; li += gridDim.x) {
    const int64_t k = list[li];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) bins[i] = 0ull;
    __syncthreads();
    for (int64_t t = threadIdx.x; t < T; t += blockDim.x) {
      const uint32_t h = X[t * ldx + k];
      const uint32_t e = (h >> 7) & 255u, m = h & 127u;
      if (e == 255u) continue;  // inf / NaN: outside the contract
      const uint32_t M = e ? (128u + m) : m;
      atomicAdd(&bins[e ? e : 1u], (unsigned long long)(M * M));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      if (accumulate) {
        const uint32_t b = __float_as_uint(I[k]);
        const uint32_t e = (b >> 23) & 255u, m = b & 0x7fffffu;
        if (e != 255u && !(b >> 31)) {
          const uint32_t M = e ? (m | 0x800000u) : m;
          const int p0 = (int)(e ? e : 1u) + 118;  // value = M * 2^(p0 - 268)
          bins[p0 >> 1] += (unsigned long long)M << (p0 & 1);
        }
      }
      I[k] = exact_bins_to_f32(bins);
    }
    __syncthreads();
  }
}

cudaError_t launch_importance(const uint16_t* X, int64_t T, int64_t K, int64_t ldx,
                              uint32_t flags, float* I, void* ws, cudaStream_t st) {
  const ImportancePlan p = plan_importance(T, K);
  double* partial = reinterpret_cast<double*>(ws);
  int32_t* list = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws) + p.partial_bytes);
  int32_t* nlist = list + K;
  const int accumulate = (flags & AAAC_IMPORTANCE_ACCUMULATE) ? 1 : 0;
  const int force_exact = (flags & AAAC_IMPORTANCE_EXACT) ? 1 : 0;
  // Height of the fp64 summation tree: a lane's running sum over its rows,
  // the fixed-order combine of the block's warps, the fixed-order combine of
  // the row blocks, and the accumulated input.
  const int64_t rows_per_lane = (p.rows_per_rb + kWarps - 1) / kWarps;
  const double d = (double)(rows_per_lane + kWarps + p.rb + 2);
  const double u = ldexp(1.0, -53);
  const double gam = d * u / (1.0 - d * u) * (1.0 + ldexp(1.0, -20));
  const double slack = (double)(T + 1) * ldexp(1.0, -248);
  cudaMemsetAsync(nlist, 0, sizeof(int32_t), st);
  importance_partial<<<dim3(p.ncb, p.rb), kThreads, 0, st>>>(X, T, K, ldx, p.rows_per_rb,
                                                             partial);
  importance_finalize<<<(unsigned)((K + 255) / 256), 256, 0, st>>>(
      partial, p.rb, K, accumulate, I, gam, slack, force_exact, list, nlist);
  importance_exact<<<128, kThreads, 0, st>>>(X, T, ldx, accumulate, I, list, nlist);
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace aaac
