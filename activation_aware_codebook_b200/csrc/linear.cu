// linear.cu -- inference on the packed format: bf16 dequantisation and the
// W4A16 linear layer.
//
// "Technical summary: AAAC", section 1 (the dequantised values from the table
// decide the weights used at inference; weight-only W4A16) and section 2, core
// mechanism 3 (BF16 tables of 16 / 15 entries; the group's choice in the sign
// bit of its positive scale, or in a bitmask when S < g):
//   W_hat[n][k] = bf16_RN(s[n][k/g] * T_bf16[c][code[n][k]])
// The product of two bf16-representable values has at most 16 significant
// bits; the bf16x2 multiply rounds the exact product once, which is that
// definition.
//
//   dequant_kernel  16 weights per thread: 8 bytes of codes in, 32 bytes of
//                   bf16 out; the 32-entry table sits in shared memory.
//   gemv_kernel     small M: a warp owns R output rows and walks K, 8 columns
//                   per lane per step; each lane expands its 8 codes (table
//                   lookup, bf16x2 scale multiply) and accumulates with fp32x2
//                   FMAs against the token tile's activations held in
//                   registers.  MT tokens x R rows = 8 accumulator pairs.
#include "common.cuh"
#include "internal.h"

namespace aaac {

namespace {

// Stored scale of group gi: bf16 bits of its magnitude, and its sign bit.
template <int FMT>
__device__ __forceinline__ uint32_t scale_bf16(const void* tagged, int64_t gi, uint32_t* tag) {
  if (FMT == kInt4) {
    const uint32_t h = __ldg(reinterpret_cast<const unsigned short*>(tagged) + gi);
    *tag = h >> 15;
    return h & 0x7fffu;
  } else {
    const uint32_t v = __ldg(reinterpret_cast<const unsigned char*>(tagged) + gi);
    *tag = v >> 7;
    // E4M3 magnitudes are exact in bf16 (3 mantissa bits, exponents 2^-9..2^8)
    return __float_as_uint(e4m3_mag(v & 0x7fu)) >> 16;
  }
}

// Choice of the selection group holding column k of row n.
__device__ __forceinline__ uint32_t group_choice(uint32_t tag, const uint8_t* cbits, int64_t n,
                                                 int nb, int k, int g, int S) {
  if (S == g) return tag;
  const int j = k / S;
  return (__ldg(cbits + n * nb + (j >> 3)) >> (j & 7)) & 1u;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

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
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// Eight dequantised weights (bf16x2 pairs, even column low) of one lane.
__device__ __forceinline__ void expand8(uint32_t cw, uint32_t sbf, uint32_t c,
                                        const unsigned short* sT, uint32_t out[4]) {
  const uint32_t s2 = sbf | (sbf << 16);
  const unsigned short* t = sT + c * 16;
#pragma unroll
  for (int p = 0; p < 4; p++) {
    const uint32_t lo = t[(cw >> (8 * p)) & 15u];
    const uint32_t hi = t[(cw >> (8 * p + 4)) & 15u];
    out[p] = bf16x2_mul(lo | (hi << 16), s2);
  }
}

template <int FMT>
__global__ void __launch_bounds__(256)
dequant_kernel(const uint8_t* __restrict__ codes, const void* __restrict__ tagged,
               const uint8_t* __restrict__ cbits, const uint16_t* __restrict__ Tb, int64_t N,
               int K, int g, int S, uint16_t* __restrict__ W_hat) {
  __shared__ unsigned short sT[32];
  if (threadIdx.x < 32) sT[threadIdx.x] = Tb[threadIdx.x];
  __syncthreads();
  const int G = K / g, nb = (K / S + 7) / 8, per_row = K / 16;
  const int64_t total = N * per_row;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = i / per_row;
    const int k0 = (int)(i - n * per_row) * 16;
    const uint2 cw = __ldg(reinterpret_cast<const uint2*>(codes + (n * K + k0) / 2));
    uint32_t out[8];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int k = k0 + 8 * h;
      uint32_t tag;
      const uint32_t sbf = scale_bf16<FMT>(tagged, n * G + k / g, &tag);
      const uint32_t c = group_choice(tag, cbits, n, nb, k, g, S);
      expand8(h ? cw.y : cw.x, sbf, c, sT, out + 4 * h);
    }
    uint4* dst = reinterpret_cast<uint4*>(W_hat + n * K + k0);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

constexpr int kGemvWarps = 4;

template <int FMT, int MT, int R>
__global__ void __launch_bounds__(kGemvWarps * 32)
gemv_kernel(const uint16_t* __restrict__ X, int M, int ldx, const uint8_t* __restrict__ codes,
            const void* __restrict__ tagged, const uint8_t* __restrict__ cbits,
            const uint16_t* __restrict__ Tb, int N, int K, int g, int S, float* __restrict__ Y) {
  __shared__ unsigned short sT[32];
  if (threadIdx.x < 32) sT[threadIdx.x] = Tb[threadIdx.x];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = (blockIdx.y * kGemvWarps + warp) * R;  // grid: x = token tiles, y = rows
  const int m0 = blockIdx.x * MT;
  if (n0 >= N) return;  // warp-uniform
  const int G = K / g, nb = (K / S + 7) / 8;
  unsigned long long acc[R][MT];
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int m = 0; m < MT; m++) acc[r][m] = 0ull;

  for (int k0 = lane * 8; k0 < K; k0 += 256) {
    unsigned long long x2[MT][4];
#pragma unroll
    for (int m = 0; m < MT; m++) {
      uint4 xv = make_uint4(0u, 0u, 0u, 0u);
      if (m0 + m < M) xv = __ldg(reinterpret_cast<const uint4*>(X + (int64_t)(m0 + m) * ldx + k0));
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int p = 0; p < 4; p++) x2[m][p] = f2pack(bf16_lo(xw[p]), bf16_hi(xw[p]));
    }
    uint32_t cw[R];
#pragma unroll
    for (int r = 0; r < R; r++)
      cw[r] = (n0 + r < N)
                  ? __ldg(reinterpret_cast<const uint32_t*>(codes + ((int64_t)(n0 + r) * K + k0) / 2))
                  : 0u;
#pragma unroll
    for (int r = 0; r < R; r++) {
      const int n = n0 + r;
      if (n >= N) break;  // warp-uniform
      uint32_t tag;
      const uint32_t sbf = scale_bf16<FMT>(tagged, (int64_t)n * G + k0 / g, &tag);
      const uint32_t c = group_choice(tag, cbits, n, nb, k0, g, S);
      uint32_t w[4];
      expand8(cw[r], sbf, c, sT, w);
#pragma unroll
      for (int p = 0; p < 4; p++) {
        const unsigned long long wf = f2pack(bf16_lo(w[p]), bf16_hi(w[p]));
#pragma unroll
        for (int m = 0; m < MT; m++) acc[r][m] = f2fma(x2[m][p], wf, acc[r][m]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int m = 0; m < MT; m++) {
      const float2 a = f2unpack(acc[r][m]);
      float v = __fadd_rn(a.x, a.y);
      for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0 && n0 + r < N && m0 + m < M) Y[(int64_t)(m0 + m) * N + n0 + r] = v;
    }
}

template <int FMT, int MT, int R>
void launch_gemv_t(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                   const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                   int64_t K, int g, int S, float* Y, cudaStream_t st) {
  const unsigned rows_per_block = kGemvWarps * R;
  // token tiles along x (consecutive blocks reuse the same codes from L2)
  const dim3 grid((unsigned)((M + MT - 1) / MT), (unsigned)((N + rows_per_block - 1) / rows_per_block));
  gemv_kernel<FMT, MT, R><<<grid, kGemvWarps * 32, 0, st>>>(X, (int)M, (int)ldx, codes, tagged,
                                                            cbits, Tb, (int)N, (int)K, g, S, Y);
}

template <int FMT>
void launch_gemv(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                 const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                 int64_t K, int g, int S, float* Y, cudaStream_t st) {
  if (M == 1) launch_gemv_t<FMT, 1, 8>(X, M, ldx, codes, tagged, cbits, Tb, N, K, g, S, Y, st);
  else if (M == 2) launch_gemv_t<FMT, 2, 4>(X, M, ldx, codes, tagged, cbits, Tb, N, K, g, S, Y, st);
  else if (M <= 4) launch_gemv_t<FMT, 4, 2>(X, M, ldx, codes, tagged, cbits, Tb, N, K, g, S, Y, st);
  else launch_gemv_t<FMT, 8, 1>(X, M, ldx, codes, tagged, cbits, Tb, N, K, g, S, Y, st);
}

}  // namespace

cudaError_t launch_dequant(const uint8_t* codes, const void* tagged, const uint8_t* cbits,
                           const uint16_t* Tb, int64_t N, int64_t K, int fmt, int g, int S,
                           uint16_t* W_hat, cudaStream_t st) {
  const int64_t chunks = N * (K / 16);
  int64_t blocks = (chunks + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  if (fmt == kInt4)
    dequant_kernel<kInt4><<<(unsigned)blocks, 256, 0, st>>>(codes, tagged, cbits, Tb, N, (int)K,
                                                            g, S, W_hat);
  else
    dequant_kernel<kNvfp4><<<(unsigned)blocks, 256, 0, st>>>(codes, tagged, cbits, Tb, N, (int)K,
                                                             g, S, W_hat);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_linear(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                          const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                          int64_t K, int fmt, int g, int S, float* Y, cudaStream_t st) {
  if (fmt == kInt4) launch_gemv<kInt4>(X, M, ldx, codes, tagged, cbits, Tb, N, K, g, S, Y, st);
  else launch_gemv<kNvfp4>(X, M, ldx, codes, tagged, cbits, Tb, N, K, g, S, Y, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace aaac
