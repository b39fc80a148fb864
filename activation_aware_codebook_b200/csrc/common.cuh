// common.cuh -- device helpers shared by the libaaac kernels (sm_100a).
//
// Number formats, IEEE total-order keys, and the per-codebook assignment
// tables: sorted codebook -> distinct values -> exact midpoint thresholds.
// "Technical summary: AAAC" section 2, core mechanism 4 (assign each weight to
// its nearest entry; 1-D Voronoi cells).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "aaac.h"

namespace aaac {

// Checked builds (compiled with -DAAAC_CHECKS, `build.py --checks`): kernels
// test the indices they compute and record the first failed check -- its
// code in the low byte, the offending value above it -- in g_check_fail,
// which aaac_device_checks reads.  No trap: the kernel goes on (a debugging
// aid for cases known to stay in bounds).  In normal builds the checks
// compile to nothing and the flag stays 0.
#ifdef AAAC_CHECKS
// one flag per translation unit (the library is built without relocatable
// device code); each unit that checks exposes it through a reader
static __device__ unsigned int g_check_fail = 0;
static inline cudaError_t read_check_flag(unsigned int* out) {
  return cudaMemcpyFromSymbol(out, g_check_fail, sizeof(unsigned int));
}
#define AAAC_CHECK(cond, code, value)                                                   \
  do {                                                                                  \
    if (!(cond)) atomicCAS(&::aaac::g_check_fail, 0u, ((unsigned)(value) << 8) | (code)); \
  } while (0)
#else
#define AAAC_CHECK(cond, code, value) \
  do {                                \
  } while (0)
#endif

constexpr int kInt4 = 0;
constexpr int kNvfp4 = 1;
constexpr int kNvfp4G = 2;            // NVFP4 with a per-tensor fp32 scale
constexpr int kWarps = 8;             // warps per block of the streaming kernels
constexpr int kThreads = kWarps * 32;
constexpr int kSegCols = 256;         // columns a warp covers per row (32 lanes x 8)
constexpr double kMagic = 6755399441055744.0;  // 1.5 * 2^52: x + magic rounds x to an integer

__host__ __device__ inline int ncodes(int fmt) { return fmt == kInt4 ? 16 : 15; }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// E4M3 ("fn"): bias 7, 3 mantissa bits, S.1111.111 is NaN; subnormal m/8 * 2^-6.
__device__ __forceinline__ float e4m3_mag(uint32_t v) {
  uint32_t e = (v >> 3) & 15u, m = v & 7u;
  if (e == 0) return __uint2float_rn(m) * 0.001953125f;  // m * 2^-9, exact
  if (e == 15 && m == 7) return __uint_as_float(0x7fc00000u);
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Decoded magnitude of a stored scale (the sign bit, a choice tag, ignored).
template <int FMT>
__device__ __forceinline__ float load_scale(const void* scales, int64_t idx) {
  if (FMT == kInt4) {
    uint32_t h = __ldg(reinterpret_cast<const unsigned short*>(scales) + idx);
    return __uint_as_float((h & 0x7fffu) << 16);
  } else {
    uint32_t v = __ldg(reinterpret_cast<const unsigned char*>(scales) + idx);
    return e4m3_mag(v & 0x7fu);
  }
}

// The scale that multiplies a codebook value: the stored scale itself, or,
// with a per-tensor scale gs, fp32_RN(gs * s8) for the stored E4M3 factor s8.
template <int FMT>
__device__ __forceinline__ float eff_scale(float s, float gs) {
  return FMT == kNvfp4G ? __fmul_rn(gs, s) : s;
}

// r = fp32_RN(1/s); a group is live when s > 0 and r is finite.
__device__ __forceinline__ bool scale_live(float s, float* r) {
  if (!(s > 0.0f)) { *r = 0.0f; return false; }
  float rc = __frcp_rn(s);
  if (!(rc < __uint_as_float(0x7f800000u))) { *r = 0.0f; return false; }
  *r = rc;
  return true;
}

__host__ __device__ __forceinline__ uint32_t order_key_bits(uint32_t b) {
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ uint32_t order_key(float f) { return order_key_bits(__float_as_uint(f)); }
__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Assignment tables of one codebook.  With the codebook sorted ascending and
// v_0 < v_1 < ... < v_{m-1} its distinct values, the nearest entry of u (lowest
// index on a tie) is idx[c] where c = #{i : u >= thr_i} and thr_i is the
// smallest fp32 strictly above the exact midpoint (v_i + v_{i+1}) / 2.  Slots
// past m-1 thresholds hold +inf; idx/val past m-1 repeat the last value.
struct Book {
  float thr[16];
  float val[16];
  int32_t idx[16];
  int32_t m;        // number of distinct values
  int32_t pad[3];
};

// Smallest fp32 strictly greater than (a + b) / 2, exactly (a, b finite fp32).
__device__ inline float midpoint_threshold(float a, float b) {
  double x = a, y = b;
  double s = __dadd_rn(x, y);                // two-sum: s + e == a + b exactly
  double bb = __dsub_rn(s, x);
  double e = __dadd_rn(__dsub_rn(x, __dsub_rn(s, bb)), __dsub_rn(y, bb));
  double h = s * 0.5, l = e * 0.5;           // exact halving
  float f = __double2float_rn(h);
  double d = __dsub_rn((double)f, h);        // exact: f is within an ulp of h
  if (d <= l) f = nextafterf(f, __uint_as_float(0x7f800000u));
  return f;
}

// Insertion sort of t[0..n) in IEEE total order (one thread).
__device__ inline void sort_book(float* t, int n) {
  for (int i = 1; i < n; i++) {
    float v = t[i];
    uint32_t kv = order_key(v);
    int j = i - 1;
    while (j >= 0 && order_key(t[j]) > kv) { t[j + 1] = t[j]; j--; }
    t[j + 1] = v;
  }
}

// Count of thresholds <= u (branchless search over 15 sorted thresholds).
__device__ __forceinline__ int book_count(const Book& bk, float u) {
  int c = 0;
  c += (bk.thr[c + 7] <= u) ? 8 : 0;
  c += (bk.thr[c + 3] <= u) ? 4 : 0;
  c += (bk.thr[c + 1] <= u) ? 2 : 0;
  c += (bk.thr[c] <= u) ? 1 : 0;
  return c;
}

}  // namespace aaac
