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
// definition.  With a per-tensor scale gs (NVFP4 variant) the scale is
// fp32_RN(gs * s8) and the value bf16_RN(fp32_RN(scale * T)): an fp32
// multiply, then the bf16x2 conversion.
//
//   dequant_kernel  one warp per row, 16 weights per lane per step: 8 bytes
//                   of codes in, 32 bytes of bf16 out; the 32-entry table
//                   sits in shared memory.
//   gemv_kernel     small M: a warp owns R output rows and MT tokens and walks
//                   K, 16 columns per lane per step; each lane expands its
//                   codes (table lookup, bf16x2 scale multiply) and
//                   accumulates with fp32x2 FMAs against the token tile's
//                   activations held in registers.
#include "common.cuh"
#include "internal.h"

namespace aaac {

namespace {

// A stored scale (bf16 bits for INT4, an E4M3 byte for NVFP4): bf16 bits of
// its magnitude, and its sign bit in *tag.  E4M3 magnitudes are exact in bf16
// (3 mantissa bits, exponents 2^-9 .. 2^8).
template <int FMT>
__device__ __forceinline__ uint32_t decode_scale(uint32_t v, uint32_t* tag) {
  if (FMT == kInt4) {
    *tag = v >> 15;
    return v & 0x7fffu;
  }
  *tag = v >> 7;
  return __float_as_uint(e4m3_mag(v & 0x7fu)) >> 16;
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

// Eight dequantised weights (bf16x2 pairs, even column low) from one word of
// codes: the table offsets of four even and four odd nibbles are formed at
// once (byte j of ev / od = 2 * code + 32 * c, a byte offset into sT), then
// one 16-bit table load per weight and one bf16x2 multiply per pair.
__device__ __forceinline__ void expand8(uint32_t cw, uint32_t sbf, uint32_t c,
                                        const unsigned short* sT, uint32_t out[4]) {
  const uint32_t s2 = sbf | (sbf << 16);
  const uint32_t cb = c ? 0x20202020u : 0u;
  const uint32_t ev = ((cw << 1) & 0x1e1e1e1eu) | cb;
  const uint32_t od = ((cw >> 3) & 0x1e1e1e1eu) | cb;
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(sT);
#pragma unroll
  for (int p = 0; p < 4; p++) {
    const uint32_t lo = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(ev, 0u, 0x4440u + p));
    const uint32_t hi = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(od, 0u, 0x4440u + p));
    out[p] = bf16x2_mul(__byte_perm(lo, hi, 0x5410u), s2);
  }
}

// expand8 with an fp32 scale (NVFP4 with a per-tensor scale): each product
// is rounded to fp32 and then to bf16, bf16_RN(fp32_RN(se * T)).
__device__ __forceinline__ void expand8g(uint32_t cw, float se, uint32_t c,
                                         const unsigned short* sT, uint32_t out[4]) {
  const uint32_t cb = c ? 0x20202020u : 0u;
  const uint32_t ev = ((cw << 1) & 0x1e1e1e1eu) | cb;
  const uint32_t od = ((cw >> 3) & 0x1e1e1e1eu) | cb;
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(sT);
#pragma unroll
  for (int p = 0; p < 4; p++) {
    const uint32_t lo = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(ev, 0u, 0x4440u + p));
    const uint32_t hi = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(od, 0u, 0x4440u + p));
    const __nv_bfloat162 r = __floats2bfloat162_rn(__fmul_rn(se, __uint_as_float(lo << 16)),
                                                   __fmul_rn(se, __uint_as_float(hi << 16)));
    out[p] = *reinterpret_cast<const uint32_t*>(&r);
  }
}

// Sixteen weights of one lane and row: codes (8 bytes), the scale of the
// group (g >= 16 holds all 16), the choice byte (S >= 8: both 8-column halves
// fall in one byte), expanded to 8 bf16x2 pairs.  gsv: the per-tensor scale
// (NVFP4 with a tensor scale only).
template <int FMT>
__device__ __forceinline__ void expand16(uint2 cw, uint32_t sv, uint32_t cbyte, int k0, int ls,
                                         bool sign_choice, const unsigned short* sT, float gsv,
                                         uint32_t out[8]) {
  uint32_t tag;
  if (FMT == kNvfp4G) {
    tag = sv >> 7;
    const float se = __fmul_rn(gsv, e4m3_mag(sv & 0x7fu));
    const uint32_t c0 = sign_choice ? tag : ((cbyte >> ((k0 >> ls) & 7)) & 1u);
    const uint32_t c1 = sign_choice ? tag : ((cbyte >> (((k0 + 8) >> ls) & 7)) & 1u);
    expand8g(cw.x, se, c0, sT, out);
    expand8g(cw.y, se, c1, sT, out + 4);
    return;
  }
  const uint32_t sbf = decode_scale<FMT>(sv, &tag);
  const uint32_t c0 = sign_choice ? tag : ((cbyte >> ((k0 >> ls) & 7)) & 1u);
  const uint32_t c1 = sign_choice ? tag : ((cbyte >> (((k0 + 8) >> ls) & 7)) & 1u);
  expand8(cw.x, sbf, c0, sT, out);
  expand8(cw.y, sbf, c1, sT, out + 4);
}

constexpr int kLinWarps = 8;

// One warp per row (rows strided over the grid); lane l covers columns
// [16 l + 512 i, +16).  Loads of a step are issued before use.
template <int FMT>
__global__ void __launch_bounds__(kLinWarps * 32)
dequant_kernel(const uint8_t* __restrict__ codes, const void* __restrict__ tagged,
               const uint8_t* __restrict__ cbits, const uint16_t* __restrict__ Tb, int N, int K,
               int lg, int ls, uint16_t* __restrict__ W_hat, const float* __restrict__ gsc) {
  __shared__ unsigned short sT[32];
  const float gsv = FMT == kNvfp4G ? __ldg(gsc) : 1.0f;
  if (threadIdx.x < 32) sT[threadIdx.x] = Tb[threadIdx.x];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = K >> lg, nb = ((K >> ls) + 7) >> 3;
  const bool sign_choice = lg == ls;
  for (int n = blockIdx.x * kLinWarps + warp; n < N; n += gridDim.x * kLinWarps) {
    const uint8_t* crow = codes + (int64_t)n * (K >> 1);
    const int64_t grow = (int64_t)n * G;
    const uint8_t* brow = cbits + (int64_t)n * nb;
    uint16_t* wrow = W_hat + (int64_t)n * K;
    // four steps' loads in flight: 45.1 -> 33.6 us on gate_proj (one step each)
#pragma unroll 4
    for (int k0 = lane * 16; k0 < K; k0 += 512) {
      const uint2 cw = __ldg(reinterpret_cast<const uint2*>(crow + (k0 >> 1)));
      const uint32_t sv = (FMT == kInt4)
          ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(tagged) + grow + (k0 >> lg))
          : (uint32_t)__ldg(reinterpret_cast<const unsigned char*>(tagged) + grow + (k0 >> lg));
      const uint32_t cbyte = sign_choice ? 0u : (uint32_t)__ldg(brow + (k0 >> (ls + 3)));
      uint32_t out[8];
      expand16<FMT>(cw, sv, cbyte, k0, ls, sign_choice, sT, gsv, out);
      uint4* dst = reinterpret_cast<uint4*>(wrow + k0);
      dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
      dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
  }
}

// Small M: a warp owns R rows and MT tokens and walks all of K, 16 columns
// per lane per step; activations for the step sit in registers (fp32 pairs)
// and feed fp32x2 FMAs with the expanded weights.  Lane partials meet in a
// shuffle tree.  UNR steps of K are unrolled (their loads issue together).
template <int FMT, int MT, int R, int UNR>
__global__ void __launch_bounds__(kLinWarps * 32)
gemv_kernel(const uint16_t* __restrict__ X, int M, int ldx, const uint8_t* __restrict__ codes,
            const void* __restrict__ tagged, const uint8_t* __restrict__ cbits,
            const uint16_t* __restrict__ Tb, int N, int K, int lg, int ls, float* __restrict__ Y,
            const float* __restrict__ gsc) {
  __shared__ unsigned short sT[32];
  const float gsv = FMT == kNvfp4G ? __ldg(gsc) : 1.0f;
  if (threadIdx.x < 32) sT[threadIdx.x] = Tb[threadIdx.x];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = (blockIdx.y * kLinWarps + warp) * R;  // grid: x = token tiles, y = row tiles
  const int m0 = blockIdx.x * MT;
  if (n0 >= N) return;  // warp-uniform
  const int G = K >> lg, nb = ((K >> ls) + 7) >> 3;
  const bool sign_choice = lg == ls;
  unsigned long long acc[R][MT];
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int m = 0; m < MT; m++) acc[r][m] = 0ull;

#pragma unroll UNR
  for (int k0 = lane * 16; k0 < K; k0 += 512) {
    uint4 xv[MT][2];
    uint2 cw[R];
    uint32_t sv[R], cbyte[R];
#pragma unroll
    for (int m = 0; m < MT; m++) {
      const uint4* xp = reinterpret_cast<const uint4*>(X + (int64_t)min(m0 + m, M - 1) * ldx + k0);
      xv[m][0] = __ldg(xp);
      xv[m][1] = __ldg(xp + 1);
    }
#pragma unroll
    for (int r = 0; r < R; r++) {
      const int n = min(n0 + r, N - 1);  // rows past N repeat the last row; never stored
      cw[r] = __ldg(reinterpret_cast<const uint2*>(codes + (((int64_t)n * K + k0) >> 1)));
      const int64_t gi = (int64_t)n * G + (k0 >> lg);
      sv[r] = (FMT == kInt4) ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(tagged) + gi)
                             : (uint32_t)__ldg(reinterpret_cast<const unsigned char*>(tagged) + gi);
      cbyte[r] = sign_choice ? 0u : (uint32_t)__ldg(cbits + (int64_t)n * nb + (k0 >> (ls + 3)));
    }
    unsigned long long x2[MT][8];
#pragma unroll
    for (int m = 0; m < MT; m++) {
      const uint32_t xw[8] = {xv[m][0].x, xv[m][0].y, xv[m][0].z, xv[m][0].w,
                              xv[m][1].x, xv[m][1].y, xv[m][1].z, xv[m][1].w};
#pragma unroll
      for (int p = 0; p < 8; p++) x2[m][p] = f2pack(bf16_lo(xw[p]), bf16_hi(xw[p]));
    }
#pragma unroll
    for (int r = 0; r < R; r++) {
      uint32_t w[8];
      expand16<FMT>(cw[r], sv[r], cbyte[r], k0, ls, sign_choice, sT, gsv, w);
#pragma unroll
      for (int p = 0; p < 8; p++) {
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

template <int FMT, int MT, int R, int UNR>
void launch_gemv_t(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                   const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                   int64_t K, int lg, int ls, float* Y, const float* gsc, cudaStream_t st) {
  // token tiles along x (consecutive blocks reuse the same codes from L2)
  const unsigned rows_per_block = kLinWarps * R;
  const dim3 grid((unsigned)((M + MT - 1) / MT), (unsigned)((N + rows_per_block - 1) / rows_per_block));
  gemv_kernel<FMT, MT, R, UNR><<<grid, kLinWarps * 32, 0, st>>>(
      X, (int)M, (int)ldx, codes, tagged, cbits, Tb, (int)N, (int)K, lg, ls, Y, gsc);
}

template <int FMT>
void launch_gemv(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                 const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                 int64_t K, int lg, int ls, float* Y, const float* gsc, cudaStream_t st) {
  // rows a warp and unrolled K steps as measured on gate_proj (us): 1 token
  // unrolled by 2, 29.5 -> 28.0; 2 tokens unrolled by 4, 35.8 -> 31.5; 3-4
  // tokens with two rows a warp unrolled by 2, 43.9 (one row: 53; four rows:
  // 46; one row unrolled by 2 or 4: 50)
  if (M == 1)
    launch_gemv_t<FMT, 1, 2, 2>(X, M, ldx, codes, tagged, cbits, Tb, N, K, lg, ls, Y, gsc, st);
  else if (M == 2)
    launch_gemv_t<FMT, 2, 2, 4>(X, M, ldx, codes, tagged, cbits, Tb, N, K, lg, ls, Y, gsc, st);
  else
    launch_gemv_t<FMT, 4, 2, 2>(X, M, ldx, codes, tagged, cbits, Tb, N, K, lg, ls, Y, gsc, st);
}

}  // namespace

constexpr int64_t kGemvMaxM = 4;  // token counts above this go to the tensor-core kernel

static int log2_of(int v) {
  int l = 0;
  while ((1 << l) < v) l++;
  return l;
}

cudaError_t launch_dequant(const uint8_t* codes, const void* tagged, const uint8_t* cbits,
                           const uint16_t* Tb, int64_t N, int64_t K, int fmt, int g, int S,
                           uint16_t* W_hat, const float* gsc, cudaStream_t st) {
  const int lg = log2_of(g), ls = log2_of(S);
  const int64_t want = (N + kLinWarps - 1) / kLinWarps;
  const unsigned blocks = (unsigned)(want < 148 * 8 ? want : 148 * 8);
  const unsigned th = kLinWarps * 32;
  if (fmt == kInt4)
    dequant_kernel<kInt4><<<blocks, th, 0, st>>>(codes, tagged, cbits, Tb, (int)N, (int)K, lg, ls,
                                                 W_hat, gsc);
  else if (fmt == kNvfp4)
    dequant_kernel<kNvfp4><<<blocks, th, 0, st>>>(codes, tagged, cbits, Tb, (int)N, (int)K, lg,
                                                  ls, W_hat, gsc);
  else
    dequant_kernel<kNvfp4G><<<blocks, th, 0, st>>>(codes, tagged, cbits, Tb, (int)N, (int)K, lg,
                                                   ls, W_hat, gsc);
  count_launches(1);
  return cudaGetLastError();
}

int linear_path(int64_t M, int64_t N, int64_t K, int fmt, int g, int S) {
  if (gemm_small_fits(M, N, K, fmt, log2_of(g), log2_of(S))) return 1;
  return M > kGemvMaxM ? 2 : 0;
}

cudaError_t launch_linear(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                          const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                          int64_t K, int fmt, int g, int S, float* Y, const float* gsc,
                          cudaStream_t st) {
  const int lg = log2_of(g), ls = log2_of(S);
  const int path = linear_path(M, N, K, fmt, g, S);
  if (path == 1) {  // 5-32 tokens: a cluster of CTAs splits a tile's K
    const cudaError_t e =
        launch_gemm_small(X, M, ldx, codes, tagged, cbits, Tb, N, K, fmt, lg, ls, Y, gsc, st);
    if (e == cudaSuccess) count_launches(1);
    return e;
  }
  if (path == 2) {  // tensor cores: dequantised tiles in shared memory
    const cudaError_t e =
        launch_gemm(X, M, ldx, codes, tagged, cbits, Tb, N, K, fmt, lg, ls, Y, gsc, st);
    if (e == cudaSuccess) count_launches(1);
    return e;
  }
  if (fmt == kInt4)
    launch_gemv<kInt4>(X, M, ldx, codes, tagged, cbits, Tb, N, K, lg, ls, Y, gsc, st);
  else if (fmt == kNvfp4)
    launch_gemv<kNvfp4>(X, M, ldx, codes, tagged, cbits, Tb, N, K, lg, ls, Y, gsc, st);
  else
    launch_gemv<kNvfp4G>(X, M, ldx, codes, tagged, cbits, Tb, N, K, lg, ls, Y, gsc, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace aaac
