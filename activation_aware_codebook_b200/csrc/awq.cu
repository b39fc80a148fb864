// awq.cu -- AWQ-style pre-scaling of a layer before the fit, and the device
// side of the grid search over the scaling exponent.
//
// "Technical summary: AAAC", section 4: AAAC combines with AWQ, which scales
// the weights before quantisation.  The page gives no formula; the scaling
// taken here (channel statistic v_k = I_k / tokens, the mean x^2 that the
// importance pass already produced):
//   p_k  = v_k^(j/32) for alpha = j/16: the product, in ascending i, of
//          v^(2^(i-5)) over the set bits i of j, each power from repeated
//          fp64 square roots;
//   z    = sqrt(max p * min p) over live channels (I_k > 0);
//   c_k  = fp32_RN(p_k / z), 1 for dead channels;
//   I'_k = fp32_RN(I_k / c_k^2)      (fp64; c_k^2 is exact);
//   W'   = bf16_RN(fp32_RN(w * c_k)).
// Every step is one correctly rounded IEEE operation (sqrt, mul, div, one
// narrowing), so the results do not depend on a math library's pow.
//
//   awq_scales_kernel   one cluster of 8 blocks: the K channel scales and the
//                       rescaled importance (two sweeps over K; the max /
//                       min between them is exact in any order and is
//                       combined over distributed shared memory).
//   awq_weights_kernel  streams W once: 16 bytes in, 16 bytes out per 8
//                       weights, c read through the read-only path.
//   awq_keep_kernel     after candidate j is packed: when its err_final beats
//                       the best earlier candidate (strictly, first minimum
//                       wins), copy its packed layer and scales to the
//                       outputs.  Every block takes the same decision from
//                       values no block writes, so there is no race.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace aaac {

namespace {

__device__ __forceinline__ double awq_power(double v, int j) {
  double q[5];
  q[4] = __dsqrt_rn(v);
#pragma unroll
  for (int i = 3; i >= 0; i--) q[i] = __dsqrt_rn(q[i + 1]);
  double p = 1.0;
#pragma unroll
  for (int i = 0; i < 5; i++)
    if ((j >> i) & 1) p = __dmul_rn(p, q[i]);
  return p;
}

constexpr int kScaleThreads = 512;
constexpr int kScaleCluster = 8;  // blocks of one cluster share the max / min over DSMEM

// Reduce (max, min, any) of the live channels' p over a warp.
__device__ __forceinline__ void reduce_live(double& pmax, double& pmin, int& any) {
  for (int o = 16; o; o >>= 1) {
    const double omax = __shfl_xor_sync(0xffffffffu, pmax, o);
    const double omin = __shfl_xor_sync(0xffffffffu, pmin, o);
    const int oany = __shfl_xor_sync(0xffffffffu, any, o);
    if (oany) {
      pmax = any ? fmax(pmax, omax) : omax;
      pmin = any ? fmin(pmin, omin) : omin;
      any = 1;
    }
  }
}

// One cluster of kScaleCluster blocks: each block takes every
// (kScaleCluster * kScaleThreads)-th channel from its offset, reduces its
// live max / min in shared memory, and every block then reads all blocks'
// partials over distributed shared memory in rank order, so all of them
// form the same z.
__global__ void __cluster_dims__(kScaleCluster, 1, 1) __launch_bounds__(kScaleThreads)
awq_scales_kernel(const float* __restrict__ I, int K, double tokens, int j, float* __restrict__ c,
                  float* __restrict__ Is) {
  __shared__ double s_max[kScaleThreads / 32], s_min[kScaleThreads / 32];
  __shared__ int s_any[kScaleThreads / 32];
  __shared__ double s_z;
  cg::cluster_group cluster = cg::this_cluster();
  const int first = (int)cluster.block_rank() * kScaleThreads + threadIdx.x;
  const int step = kScaleCluster * kScaleThreads;
  double pmax = 0.0, pmin = 0.0;
  int any = 0;
  for (int k = first; k < K; k += step) {
    const float ik = I[k];
    if (!(ik > 0.0f)) continue;
    const double p = awq_power(__ddiv_rn((double)ik, tokens), j);
    if (!any || p > pmax) pmax = p;
    if (!any || p < pmin) pmin = p;
    any = 1;
  }
  reduce_live(pmax, pmin, any);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_max[warp] = pmax;
    s_min[warp] = pmin;
    s_any[warp] = any;
  }
  __syncthreads();
  if (warp == 0) {  // the block's partial, left in slot 0
    pmax = lane < kScaleThreads / 32 ? s_max[lane] : 0.0;
    pmin = lane < kScaleThreads / 32 ? s_min[lane] : 0.0;
    any = lane < kScaleThreads / 32 ? s_any[lane] : 0;
    reduce_live(pmax, pmin, any);
    __syncwarp();
    if (lane == 0) {
      s_max[0] = pmax;
      s_min[0] = pmin;
      s_any[0] = any;
    }
  }
  cluster.sync();  // every block's partial is in its shared memory
  if (threadIdx.x == 0) {
    double mx = 0.0, mn = 0.0;
    int a = 0;
    for (int r = 0; r < kScaleCluster; r++) {
      const int ra = *cluster.map_shared_rank(&s_any[0], r);
      if (!ra) continue;
      const double rmax = *cluster.map_shared_rank(&s_max[0], r);
      const double rmin = *cluster.map_shared_rank(&s_min[0], r);
      mx = a ? fmax(mx, rmax) : rmax;
      mn = a ? fmin(mn, rmin) : rmin;
      a = 1;
    }
    s_z = a ? __dsqrt_rn(__dmul_rn(mx, mn)) : 1.0;
  }
  cluster.sync();  // no block leaves while another still reads its partial
  const double z = s_z;
  for (int k = first; k < K; k += step) {
    const float ik = I[k];
    if (!(ik > 0.0f)) {
      c[k] = 1.0f;
      Is[k] = ik;
      continue;
    }
    const double p = awq_power(__ddiv_rn((double)ik, tokens), j);
    const float ck = __double2float_rn(__ddiv_rn(p, z));
    const double cc = __dmul_rn((double)ck, (double)ck);
    c[k] = ck;
    Is[k] = __double2float_rn(__ddiv_rn((double)ik, cc));
  }
}

__device__ __forceinline__ uint32_t scale_pair(uint32_t w2, float c0, float c1) {
  const __nv_bfloat162 r =
      __floats2bfloat162_rn(__fmul_rn(bf16_lo(w2), c0), __fmul_rn(bf16_hi(w2), c1));
  return *reinterpret_cast<const uint32_t*>(&r);
}

__global__ void __launch_bounds__(kThreads)
awq_weights_kernel(const uint4* __restrict__ W, uint32_t n_vec, uint32_t k_vec,
                   const float4* __restrict__ c, uint4* __restrict__ Wout) {
  for (uint32_t i = blockIdx.x * kThreads + threadIdx.x; i < n_vec; i += gridDim.x * kThreads) {
    const uint32_t v = i % k_vec;
    const uint4 w = __ldcs(W + i);
    const float4 ca = __ldg(c + 2 * v), cb = __ldg(c + 2 * v + 1);
    uint4 o;
    o.x = scale_pair(w.x, ca.x, ca.y);
    o.y = scale_pair(w.y, ca.z, ca.w);
    o.z = scale_pair(w.z, cb.x, cb.y);
    o.w = scale_pair(w.w, cb.z, cb.w);
    __stcs(Wout + i, o);
  }
}

constexpr int kKeepSegs = 6;

struct KeepArgs {
  const unsigned char* src[kKeepSegs];
  unsigned char* dst[kKeepSegs];
  size_t bytes[kKeepSegs];
  int segs;
  int j;
  const double* err_alpha;
  double* err_final;
  int32_t* best;
};

__global__ void __launch_bounds__(kThreads) awq_keep_kernel(KeepArgs a) {
  // the best earlier candidate, first minimum, as the host-side search keeps it
  int b = 0;
  for (int i = 1; i < a.j; i++)
    if (a.err_alpha[i] < a.err_alpha[b]) b = i;
  const bool better = (a.j == 0) || (a.err_alpha[a.j] < a.err_alpha[b]);
  if (!better) return;
  const size_t tid = (size_t)blockIdx.x * kThreads + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * kThreads;
  for (int s = 0; s < a.segs; s++) {
    const size_t n16 = a.bytes[s] / 16;
    const uint4* src = reinterpret_cast<const uint4*>(a.src[s]);
    uint4* dst = reinterpret_cast<uint4*>(a.dst[s]);
    for (size_t i = tid; i < n16; i += stride) dst[i] = src[i];
    for (size_t i = n16 * 16 + tid; i < a.bytes[s]; i += stride) a.dst[s][i] = a.src[s][i];
  }
  if (tid == 0) {
    if (a.err_final) *a.err_final = a.err_alpha[a.j];
    if (a.best) *a.best = a.j;
  }
}

}  // namespace

cudaError_t launch_awq_prescale(const uint16_t* W, int64_t N, int64_t K, const float* I,
                                int64_t tokens, int j, float* c, float* Is, uint16_t* Wout,
                                cudaStream_t st) {
  awq_scales_kernel<<<kScaleCluster, kScaleThreads, 0, st>>>(I, (int)K, (double)tokens, j, c, Is);
  const uint32_t n_vec = (uint32_t)(N * K / 8), k_vec = (uint32_t)(K / 8);
  int blocks = (int)((n_vec + kThreads - 1) / kThreads);
  if (blocks > 148 * 8) blocks = 148 * 8;
  awq_weights_kernel<<<blocks, kThreads, 0, st>>>(
      reinterpret_cast<const uint4*>(W), n_vec, k_vec, reinterpret_cast<const float4*>(c),
      reinterpret_cast<uint4*>(Wout));
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t launch_awq_keep(int j, const double* err_alpha, const void* const* src,
                            void* const* dst, const size_t* bytes, int segs, double* err_final,
                            int32_t* best, cudaStream_t st) {
  KeepArgs a{};
  size_t total = 0;
  for (int s = 0; s < segs && s < kKeepSegs; s++) {
    if (bytes[s] == 0) continue;  // absent output (no choice bits, no tensor scale)
    a.src[a.segs] = static_cast<const unsigned char*>(src[s]);
    a.dst[a.segs] = static_cast<unsigned char*>(dst[s]);
    a.bytes[a.segs] = bytes[s];
    total += bytes[s];
    a.segs++;
  }
  a.j = j;
  a.err_alpha = err_alpha;
  a.err_final = err_final;
  a.best = best;
  int blocks = (int)((total / 16 + kThreads - 1) / kThreads);
  if (blocks < 1) blocks = 1;
  if (blocks > 148 * 4) blocks = 148 * 4;
  awq_keep_kernel<<<blocks, kThreads, 0, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace aaac
