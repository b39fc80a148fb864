// gemm.cu -- the W4A16 linear above 4 tokens on the 5th-generation tensor
// cores: Y[m][n] = sum_k X[m][k] * W_hat[n][k] with W_hat expanded from the
// packed format tile by tile in shared memory.  Three kernels: gemm_kernel
// (the fused expansion, below), gemm_small_kernel (5 to 32 tokens: a cluster
// of 2 to 8 CTAs splits K, codes by TMA), and gemm_tma_kernel (dequantised
// weights, a persistent TMA-fed GEMM for 192 tokens and more).
//
// "Technical summary: AAAC", section 1 (weight-only W4A16 inference: the
// dequantised values from the tables decide the weights used) and section 2,
// core mechanism 3 (BF16 tables, the choice in the scale's sign bit or a
// bitmask).  W_hat[n][k] = bf16_RN(s * T_c[code]) exactly as aaac_dequant.
//
// One CTA computes a 128 (weight rows) x BT (tokens) tile of Y^T:
//   D[n][t] += A[n][k] * B[t][k],  A = W_hat tile, B = X tile, both K-major,
// with tcgen05.mma kind::f16 (bf16 in, fp32 accumulate in TMEM).  Per 64-wide
// K block (one 128-byte swizzle row per operand row):
//   warp 0      one lane issues the TMA load of the X tile (SWIZZLE_128B) into
//               stage s (a plain copy into this CTA only);
//   warps 2..9  256 producer threads, two per weight row (32 columns each):
//               16 bytes of codes, the scales and the
//               choice byte, loaded up to 2 x kPre stages ahead into two
//               alternating register sets -> bf16 values written in
//               the 128B-swizzled K-major layout, made visible to the tensor
//               core with fence.proxy.async, then an arrive on the stage
//               barrier;
//   warp 1      allocates TMEM (BT fp32 columns); one lane issues 4 MMAs
//               (K = 16 each) per stage and commits them to the stage's
//               "empty" barrier, and after the last stage to "accumulator full";
//   epilogue    warps 2..9 read their TMEM lane quadrant (rows; two warps per
//               quadrant, one half of the token columns each) with
//               tcgen05.ld 32x32b, 32 token columns at a time, and store fp32
//               Y[t][n]: for each token the warp writes 32 consecutive n.
// When the tiles are fewer than the SMs, K is split in two: Y is zeroed and
// both halves add their partial tiles with float atomics (two terms onto
// zero: the result does not depend on their order).
// Every mbarrier wait is bounded by the global timer (about 2 s); a wait that
// runs out sets a device flag, the tile is written as NaN and the CTA still
// releases its TMEM.
#include <cuda.h>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace aaac {

namespace {

constexpr int kBN = 128;               // weight rows per CTA (MMA M)
constexpr int kBK = 64;                // K per stage: one 128-byte bf16 row
constexpr int kStagesG = 3;
constexpr int kPre = 2;              // producer stages loaded ahead, per register set
constexpr int kProdWarps = 8;          // producer / epilogue warps (2 .. 9)
constexpr int kGemmThreads = (2 + kProdWarps) * 32;
constexpr int kATileBytes = kBN * kBK * 2;  // 16 KB
constexpr uint64_t kWaitNs = 2000000000ull;
// A waiting thread is suspended in the barrier (no issue slots) until the
// phase completes or this many nanoseconds pass; then the time bound is
// checked and the wait is retried.
constexpr uint32_t kSuspendNs = 1000000u;

__device__ unsigned int g_gemm_timeout = 0;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of the given parity; false (and the device flag
// set) when the time bound runs out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t n = 1;; n++) {
    if (mbar_test(bar, parity)) return true;
    if ((n & 15u) == 0u && global_ns() - t0 > kWaitNs) {  // the clock every 16 tries
      atomicExch(&g_gemm_timeout, 1u);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO = 64 x 16 B), LBO = 1 (unused by swizzled K-major),
// descriptor version 1 (bit 46), layout type 2 = SWIZZLE_128B (bits 61..63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t mma_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

template <int FMT>
__device__ __forceinline__ uint32_t scale_bits(uint32_t v, uint32_t* tag) {
  if (FMT == kInt4) {
    *tag = v >> 15;
    return v & 0x7fffu;
  }
  *tag = v >> 7;
  return __float_as_uint(e4m3_mag(v & 0x7fu)) >> 16;  // exact in bf16
}

// Eight dequantised weights (bf16x2 pairs, even column low) from one word of
// codes; byte j of ev / od = 2 * code + 32 * c indexes the bf16 table sT.
__device__ __forceinline__ uint4 expand8(uint32_t cw, uint32_t sbf, uint32_t c,
                                         const unsigned short* sT) {
  const uint32_t s2 = sbf | (sbf << 16);
  const uint32_t cb = c ? 0x20202020u : 0u;
  const uint32_t ev = ((cw << 1) & 0x1e1e1e1eu) | cb;
  const uint32_t od = ((cw >> 3) & 0x1e1e1e1eu) | cb;
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(sT);
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; p++) {
    const uint32_t lo = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(ev, 0u, 0x4440u + p));
    const uint32_t hi = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(od, 0u, 0x4440u + p));
    o[p] = bf16x2_mul(__byte_perm(lo, hi, 0x5410u), s2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// expand8 with an fp32 scale (NVFP4 with a per-tensor scale):
// bf16_RN(fp32_RN(se * T)) per weight.
__device__ __forceinline__ uint4 expand8g(uint32_t cw, float se, uint32_t c,
                                          const unsigned short* sT) {
  const uint32_t cb = c ? 0x20202020u : 0u;
  const uint32_t ev = ((cw << 1) & 0x1e1e1e1eu) | cb;
  const uint32_t od = ((cw >> 3) & 0x1e1e1e1eu) | cb;
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(sT);
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; p++) {
    const uint32_t lo = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(ev, 0u, 0x4440u + p));
    const uint32_t hi = *reinterpret_cast<const unsigned short*>(tb + __byte_perm(od, 0u, 0x4440u + p));
    const __nv_bfloat162 r = __floats2bfloat162_rn(__fmul_rn(se, __uint_as_float(lo << 16)),
                                                   __fmul_rn(se, __uint_as_float(hi << 16)));
    o[p] = *reinterpret_cast<const uint32_t*>(&r);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

struct GemmArgs {
  const uint8_t* codes;
  const void* tagged;
  const uint8_t* cbits;
  const uint16_t* Tb;
  float* Y;
  int M, N, K, lg, ls;
  int split;  // 1: one CTA per tile; 2: two K halves added into a zeroed Y
  const float* gsc;  // per-tensor scale (NVFP4 with a tensor scale only)
};

template <int FMT, int BT>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap xmap, GemmArgs a) {
  extern __shared__ __align__(1024) unsigned char gsm[];
  // 1024-byte aligned operand stages (the swizzle atom), then the barriers
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(gsm) + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = base;                                   // kStagesG x 16 KB
  unsigned char* sB = base + kStagesG * kATileBytes;          // kStagesG x BT*128
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStagesG * BT * 128);
  uint64_t* empty = full + kStagesG;
  uint64_t* accum = empty + kStagesG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  __shared__ unsigned short sT[32];
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN, t0 = blockIdx.y * BT;
  // K blocks of this CTA: all, or one half when the tile is split over K
  const int nkb_all = (a.K + kBK - 1) / kBK;
  const int kb_lo = a.split == 2 ? (blockIdx.z ? (nkb_all + 1) / 2 : 0) : 0;
  const int nkb = a.split == 2 ? (blockIdx.z ? nkb_all - kb_lo : (nkb_all + 1) / 2) : nkb_all;

  if (threadIdx.x < 32) sT[threadIdx.x] = a.Tb[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesG; s++) {
      mbar_init(&full[s], 1 + kProdWarps);  // TMA expect_tx + producer warps
      mbar_init(&empty[s], 1);     // MMA commit
    }
    mbar_init(accum, 1);
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(BT));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // X tiles by TMA
      int issued = 0;
      for (int kb = 0; kb < nkb; kb++) {
        const int s = kb % kStagesG;
        const uint32_t wrap = kb / kStagesG;
        if (kb >= kStagesG && !mbar_wait(&empty[s], (wrap - 1) & 1)) { s_fail = 1; break; }
        mbar_arrive_expect_tx(&full[s], BT * 128);
        tma_load_2d(sB + s * BT * 128, &xmap, &full[s], (kb_lo + kb) * kBK, t0);
        issued = kb + 1;
      }
      // the last copies have landed before the CTA can exit (bounded)
      for (int kb = issued > kStagesG ? issued - kStagesG : 0; kb < issued; kb++)
        if (!mbar_wait(&full[kb % kStagesG], (kb / kStagesG) & 1)) { s_fail = 1; break; }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issue
      const uint32_t idesc = mma_idesc(kBN, BT);
      for (int kb = 0; kb < nkb; kb++) {
        const int s = kb % kStagesG;
        if (!mbar_wait(&full[s], (kb / kStagesG) & 1)) { s_fail = 1; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kATileBytes), b0 = smem_u32(sB + s * BT * 128);
#pragma unroll
        for (int k = 0; k < kBK / 16; k++)
          mma_bf16(tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
        mma_commit(&empty[s]);  // stage s free once these MMAs completed
      }
      mma_commit(accum);
    }
  } else {
    // producers: thread p handles half h = p & 1 (32 columns) of weight row
    // r = p >> 1 of every stage.
    const int p = threadIdx.x - 64;
    const int h = p & 1;
    const int G = a.K >> a.lg, nb = ((a.K >> a.ls) + 7) >> 3;
    const bool sign_choice = a.lg == a.ls;
    const float gsv = FMT == kNvfp4G ? __ldg(a.gsc) : 1.0f;
    const int rowi = p >> 1;
    const int nrow_p = n0 + rowi;
    const bool rok = nrow_p < a.N;
    const int nn = rok ? nrow_p : 0;
    const uint8_t* crow = a.codes + (int64_t)nn * (a.K >> 1);
    const int64_t grow = (int64_t)nn * G;
    const uint8_t* brow = a.cbits + (int64_t)nn * nb;
    // raw data of kPre consecutive stages in registers; two sets alternate, so
    // the loads of stages kb + kPre .. kb + 2 kPre - 1 are in flight while
    // stages kb .. kb + kPre - 1 are expanded
    struct Raw {
      uint4 cw[kPre];
      uint32_t sv[kPre][2];
      uint32_t cb[kPre];
    };
    auto load_set = [&](Raw& R, int kb0) {
#pragma unroll
      for (int u = 0; u < kPre; u++) {
        const int k = (kb_lo + kb0 + u) * kBK + h * 32;  // first column of this row half
        const bool in = rok && k < a.K;
        // rows are K/2 bytes apart (a multiple of 8): two 8-byte loads
        uint2 c0 = make_uint2(0u, 0u), c1 = make_uint2(0u, 0u);
        if (in) {
          const uint2* src = reinterpret_cast<const uint2*>(crow + (k >> 1));
          c0 = __ldg(src);
          if (k + 16 < a.K) c1 = __ldg(src + 1);
        }
        R.cw[u] = make_uint4(c0.x, c0.y, c1.x, c1.y);
#pragma unroll
        for (int q = 0; q < 2; q++) {  // scales of columns k and k + 16 (g >= 16)
          const int kq = min(k + 16 * q, a.K - 16);
          R.sv[u][q] = !in ? 0u
              : (FMT == kInt4)
                  ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(a.tagged) + grow + (kq >> a.lg))
                  : (uint32_t)__ldg(reinterpret_cast<const unsigned char*>(a.tagged) + grow + (kq >> a.lg));
        }
        R.cb[u] = (!in || sign_choice) ? 0u : (uint32_t)__ldg(brow + (k >> (a.ls + 3)));
      }
    };
    bool ok = true;
    const uint32_t rsw = (uint32_t)(rowi & 7);
    const uint32_t roff = (uint32_t)(rowi >> 3) * 1024u + rsw * 128u;
    auto run_set = [&](const Raw& R, int kb0) {
#pragma unroll
      for (int u = 0; u < kPre; u++) {
        const int kb = kb0 + u;
        if (kb >= nkb || !ok) return;
        const int s = kb % kStagesG;
        const uint32_t wrap = kb / kStagesG;
        if (kb >= kStagesG) {  // warp-uniform outcome
          ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], (wrap - 1) & 1));
          if (!ok) {
            s_fail = 1;
            return;
          }
        }
        unsigned char* dst = sA + s * kATileBytes + roff;
        const uint32_t words[4] = {R.cw[u].x, R.cw[u].y, R.cw[u].z, R.cw[u].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const int k = (kb_lo + kb) * kBK + h * 32 + 8 * j;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (rok && k < a.K) {
            uint32_t tag;
            if (FMT == kNvfp4G) {
              const uint32_t sv = R.sv[u][j >> 1];
              tag = sv >> 7;
              const uint32_t ch = sign_choice ? tag : (R.cb[u] >> ((k >> a.ls) & 7)) & 1u;
              v = expand8g(words[j], __fmul_rn(gsv, e4m3_mag(sv & 0x7fu)), ch, sT);
            } else {
              const uint32_t sbf = scale_bits<FMT>(R.sv[u][j >> 1], &tag);
              const uint32_t ch = sign_choice ? tag : (R.cb[u] >> ((k >> a.ls) & 7)) & 1u;
              v = expand8(words[j], sbf, ch, sT);
            }
          }
          const uint32_t c = (uint32_t)(h * 4 + j);
          *reinterpret_cast<uint4*>(dst + ((c ^ rsw) << 4)) = v;
        }
        fence_proxy_async();  // generic-proxy stores -> visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      }
    };
    Raw RA, RB;
    load_set(RA, 0);
    for (int kb0 = 0; kb0 < nkb && ok; kb0 += 2 * kPre) {
      if (kb0 + kPre < nkb) load_set(RB, kb0 + kPre);
      run_set(RA, kb0);
      if (kb0 + kPre >= nkb || !ok) break;
      if (kb0 + 2 * kPre < nkb) load_set(RA, kb0 + 2 * kPre);
      run_set(RB, kb0 + kPre);
    }
    // epilogue: TMEM lane quadrant of this warp = 32 weight rows
    const bool got = __all_sync(0xffffffffu, mbar_wait(accum, 0));
    tc_fence_after();
    const int q = warp & 3;               // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;     // which half of the token columns
    const int nrow = n0 + q * 32 + lane;
    const bool fail = !got || s_fail;
    for (int j0 = half * (BT / 2); j0 < (half + 1) * (BT / 2); j0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)j0, r);
#pragma unroll
      for (int j = 0; j < 32; j++) {
        const int t = t0 + j0 + j;
        if (nrow < a.N && t < a.M) {
          float* y = a.Y + (int64_t)t * a.N + nrow;
          const float v = fail ? __int_as_float(0x7fc00000) : __uint_as_float(r[j]);
          // two partials into a zeroed Y: 0 + a + b is the same in either order
          if (a.split == 2) atomicAdd(y, v);
          else *y = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BT));
  }
}

// ---------------------------------------------------------------------------
// Large token counts: W_hat dequantised once into the caller's workspace
// (aaac_dequant's kernel), then a persistent bf16 x bf16 tcgen05 GEMM with
// both operands brought in by TMA.  The fused kernel above expands W again
// for every token tile; here the expansion is paid once.
//   one CTA per SM walks the 128 x 256 output tiles t = blockIdx.x, +grid, ...
//   (weight-row tile major, so the CTAs in flight share their W rows in L2);
//   warp 0      one lane issues the TMA loads of the W_hat tile (128 rows x 64)
//               and the X tile (256 x 64) of every stage, each into this CTA only;
//   warp 1      allocates all 512 TMEM columns: two 256-column accumulators,
//               tiles alternating between them; one lane issues the MMAs and
//               commits each tile's accumulator to acc_full[b];
//   warps 2..9  epilogue of tile i from accumulator i & 1 while the MMAs of
//               tile i + 1 run in the other one; acc_empty[b] hands it back.
// Waits are bounded as in gemm_kernel.
// ---------------------------------------------------------------------------
constexpr int kStagesT = 4;
constexpr int kBTT = 256;  // tokens per tile

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tma_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                GemmArgs a, int tiles_t, int tiles) {
  extern __shared__ __align__(1024) unsigned char gsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(gsm) + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = base;                                   // kStagesT x 16 KB
  unsigned char* sB = base + kStagesT * kATileBytes;          // kStagesT x 32 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStagesT * kBTT * 128);
  uint64_t* empty = full + kStagesT;
  uint64_t* acc_full = empty + kStagesT;   // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (a.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesT; s++) {
      mbar_init(&full[s], 1);   // the TMA thread's expect_tx
      mbar_init(&empty[s], 1);  // MMA commit
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&acc_full[b], 1);           // MMA commit of a tile
      mbar_init(&acc_empty[b], kProdWarps);  // one arrive per epilogue warp
    }
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(2 * kBTT));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // W_hat and X tiles by TMA, stage after stage across the tiles
      int it = 0;     // stage uses so far
      for (int tile = blockIdx.x; tile < tiles && !s_fail; tile += gridDim.x) {
        const int n0 = (tile / tiles_t) * kBN, t0 = (tile % tiles_t) * kBTT;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % kStagesT;
          if (it >= kStagesT && !mbar_wait(&empty[s], ((it / kStagesT) - 1) & 1)) {
            s_fail = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kATileBytes + kBTT * 128);
          tma_load_2d(sA + s * kATileBytes, &wmap, &full[s], kb * kBK, n0);
          tma_load_2d(sB + s * kBTT * 128, &xmap, &full[s], kb * kBK, t0);
        }
      }
      // the last copies have landed before the CTA can exit (bounded)
      for (int j = it > kStagesT ? it - kStagesT : 0; j < it; j++)
        if (!mbar_wait(&full[j % kStagesT], (j / kStagesT) & 1)) { s_fail = 1; break; }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issue
      const uint32_t idesc = mma_idesc(kBN, kBTT);
      int it = 0, i = 0;
      for (int tile = blockIdx.x; tile < tiles && !s_fail; tile += gridDim.x, i++) {
        const int b = i & 1;
        // the accumulator's previous tile (i - 2) has been read out
        if (i >= 2 && !mbar_wait(&acc_empty[b], ((i >> 1) - 1) & 1)) { s_fail = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * kBTT);
        bool ok = true;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % kStagesT;
          if (!mbar_wait(&full[s], (it / kStagesT) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kATileBytes), b0 = smem_u32(sB + s * kBTT * 128);
#pragma unroll
          for (int k = 0; k < kBK / 16; k++)
            mma_bf16(d, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc,
                     (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!ok) { s_fail = 1; break; }
        mma_commit(&acc_full[b]);
      }
    }
  } else {
    const int q = warp & 3;               // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;     // which half of the token columns
    int i = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, i++) {
      const int b = i & 1;
      const int n0 = (tile / tiles_t) * kBN, t0 = (tile % tiles_t) * kBTT;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], (i >> 1) & 1));
      tc_fence_after();
      const bool fail = !got || s_fail;
      const int nrow = n0 + q * 32 + lane;
      for (int j0 = half * (kBTT / 2); j0 < (half + 1) * (kBTT / 2); j0 += 32) {
        uint32_t r[32];
        if (!fail) tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kBTT + j0), r);
#pragma unroll
        for (int j = 0; j < 32; j++) {
          const int t = t0 + j0 + j;
          if (nrow < a.N && t < a.M)
            a.Y[(int64_t)t * a.N + nrow] = fail ? __int_as_float(0x7fc00000) : __uint_as_float(r[j]);
        }
      }
      if (fail) break;  // the MMA warp stopped; nothing more to read
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(2 * kBTT));
  }
}

// ---------------------------------------------------------------------------
// Small token counts (5 to 32 tokens): the work is the stream of 4-bit codes,
// so the kernel is laid out to keep HBM busy and to spend few instructions
// per weight.  A cluster of C CTAs (2 to 8, along grid y) shares one 128-row
// tile of W; CTA r of the cluster takes a contiguous 1/C of the 64-wide K
// blocks.
//   warp 0      one lane issues, per stage, the TMA copies of the code tile
//               (128 rows x 32 bytes, no swizzle) and of the X tile (BT x 64,
//               SWIZZLE_128B), each into this CTA only, on ld_full[s];
//   warp 1      allocates TMEM and issues the MMAs (M = 128, N = BT) of a
//               stage once the producers have filled it (a_full[s]), then
//               commits the stage to empty[s] and, after the last, accum;
//   warps 2..9  producers: two threads per weight row, 32 columns each;
//               codes from the stage's code tile, the row's scales and choice
//               bits from shared memory (staged once at the start), expanded
//               into the stage's swizzled bf16 A tile (expand8 as in the
//               fused kernel), then fence.proxy.async and one arrive per warp.
// The row's partial (128 x BT fp32) goes from TMEM to the CTA's shared memory;
// after a cluster barrier each CTA sums 1/C of the tile's outputs over the
// cluster's partials in rank order (distributed shared memory, fixed order:
// the result does not depend on timing) and stores Y.  A second cluster
// barrier keeps every partial alive until all CTAs have read it.  Waits on
// mbarriers are bounded as in gemm_kernel; a CTA that gives up writes NaN
// partials but still reaches both cluster barriers.
// ---------------------------------------------------------------------------
constexpr int kStagesS = 4;
constexpr int kSmallSmemMax = 227 * 1024;
constexpr int kCodeTileBytes = kBN * kBK / 2;  // 4 KB: 128 rows x 32 bytes

struct SmallArgs {
  const void* tagged;
  const uint8_t* cbits;
  const uint16_t* Tb;
  float* Y;
  int M, N, K, lg, ls;
  int nkb_all;        // 64-wide K blocks of the layer
  int sc_stride;      // shared bytes per row for its scales
  int cb_stride;      // shared bytes per row for its choice bits
  const float* gsc;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NC]);
template <>
__device__ __forceinline__ void tmem_ld_cols<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int BT>
__host__ __device__ constexpr uint32_t small_tmem_cols() {
  return BT < 32 ? 32u : (uint32_t)BT;
}

template <int FMT, int BT>
__global__ void __launch_bounds__(kGemmThreads, 2)
gemm_small_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                  SmallArgs a) {
  extern __shared__ __align__(1024) unsigned char gsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(gsm) + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = base;                                  // kStagesS x 16 KB
  unsigned char* sB = sA + kStagesS * kATileBytes;           // kStagesS x BT*128
  unsigned char* sC = sB + kStagesS * BT * 128;              // kStagesS x 4 KB
  unsigned char* sSc = sC + kStagesS * kCodeTileBytes;       // 128 x sc_stride
  unsigned char* sCb = sSc + kBN * a.sc_stride;              // 128 x cb_stride
  uint64_t* ld_full = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(sCb + kBN * a.cb_stride) + 7) & ~(uintptr_t)7);
  uint64_t* a_full = ld_full + kStagesS;
  uint64_t* empty = a_full + kStagesS;
  uint64_t* accum = empty + kStagesS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  float* P = reinterpret_cast<float*>(sA);  // the partial tile [BT][128], after the MMAs
  __shared__ unsigned short sT[32];
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank(), csize = cluster_size();
  const int n0 = blockIdx.x * kBN;
  const int kb_lo = (int)(crank * (uint32_t)a.nkb_all / csize);
  const int kb_hi = (int)((crank + 1) * (uint32_t)a.nkb_all / csize);
  const int nkb = kb_hi - kb_lo;  // >= 1: the host takes csize <= nkb_all
  const int col_lo = kb_lo * kBK;
  const int col_hi = min(a.K, kb_hi * kBK);
  const int gi_lo = col_lo >> a.lg;
  const int bb_lo = (col_lo >> a.ls) >> 3;
  const bool sign_choice = a.lg == a.ls;

  if (threadIdx.x < 32) sT[threadIdx.x] = a.Tb[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesS; s++) {
      mbar_init(&ld_full[s], 1);          // the TMA lane's expect_tx
      mbar_init(&a_full[s], kProdWarps);  // one arrive per producer warp
      mbar_init(&empty[s], 1);            // MMA commit
    }
    mbar_init(accum, 1);
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(small_tmem_cols<BT>()));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp >= 2) {
    // stage the tile rows' scales and choice bits of this CTA's K range
    const int p = threadIdx.x - 64, row = p >> 1, h = p & 1;
    const int n = n0 + row;
    const int ng = ((col_hi - 1) >> a.lg) - gi_lo + 1;
    const int G = a.K >> a.lg;
    if (FMT == kInt4) {
      const unsigned short* src = reinterpret_cast<const unsigned short*>(a.tagged) + (int64_t)n * G + gi_lo;
      unsigned short* dst = reinterpret_cast<unsigned short*>(sSc + row * a.sc_stride);
      for (int i = h; i < ng; i += 2) dst[i] = n < a.N ? __ldg(src + i) : (unsigned short)0;
    } else {
      const unsigned char* src = reinterpret_cast<const unsigned char*>(a.tagged) + (int64_t)n * G + gi_lo;
      unsigned char* dst = sSc + row * a.sc_stride;
      for (int i = h; i < ng; i += 2) dst[i] = n < a.N ? __ldg(src + i) : (unsigned char)0;
    }
    if (!sign_choice) {
      const int nb = ((a.K >> a.ls) + 7) >> 3;
      const int nbb = (((col_hi - 1) >> a.ls) >> 3) - bb_lo + 1;
      const uint8_t* src = a.cbits + (int64_t)n * nb + bb_lo;
      unsigned char* dst = sCb + row * a.cb_stride;
      for (int i = h; i < nbb; i += 2) dst[i] = n < a.N ? __ldg(src + i) : (unsigned char)0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // code and X tiles by TMA
      int issued = 0;
      for (int kb = 0; kb < nkb; kb++) {
        const int s = kb % kStagesS;
        if (kb >= kStagesS && !mbar_wait(&empty[s], ((kb / kStagesS) - 1) & 1)) { s_fail = 1; break; }
        mbar_arrive_expect_tx(&ld_full[s], BT * 128 + kCodeTileBytes);
        tma_load_2d(sB + s * BT * 128, &xmap, &ld_full[s], (kb_lo + kb) * kBK, 0);
        tma_load_2d(sC + s * kCodeTileBytes, &cmap, &ld_full[s], (kb_lo + kb) * (kBK / 2), n0);
        issued = kb + 1;
      }
      // the last copies have landed before the CTA can exit (bounded)
      for (int kb = issued > kStagesS ? issued - kStagesS : 0; kb < issued; kb++)
        if (!mbar_wait(&ld_full[kb % kStagesS], (kb / kStagesS) & 1)) { s_fail = 1; break; }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issue
      const uint32_t idesc = mma_idesc(kBN, BT);
      for (int kb = 0; kb < nkb; kb++) {
        const int s = kb % kStagesS;
        const uint32_t ph = (kb / kStagesS) & 1;
        if (!mbar_wait(&ld_full[s], ph) || !mbar_wait(&a_full[s], ph)) { s_fail = 1; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kATileBytes), b0 = smem_u32(sB + s * BT * 128);
#pragma unroll
        for (int k = 0; k < kBK / 16; k++)
          mma_bf16(tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(accum);
    }
  } else {
    // producers: thread p fills half h = p & 1 (32 columns) of weight row p >> 1
    const int p = threadIdx.x - 64;
    const int h = p & 1, rowi = p >> 1;
    const bool rok = n0 + rowi < a.N;
    const float gsv = FMT == kNvfp4G ? __ldg(a.gsc) : 1.0f;
    const uint32_t rsw = (uint32_t)(rowi & 7);
    const uint32_t roff = (uint32_t)(rowi >> 3) * 1024u + rsw * 128u;
    const unsigned char* scrow = sSc + rowi * a.sc_stride;
    const unsigned char* cbrow = sCb + rowi * a.cb_stride;
    for (int kb = 0; kb < nkb; kb++) {
      const int s = kb % kStagesS;
      if (!__all_sync(0xffffffffu, mbar_wait(&ld_full[s], (kb / kStagesS) & 1))) {
        s_fail = 1;
        break;
      }
      const uint4 cw = *reinterpret_cast<const uint4*>(sC + s * kCodeTileBytes + rowi * 32 + h * 16);
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
      unsigned char* dst = sA + s * kATileBytes + roff;
      const int k0 = (kb_lo + kb) * kBK + h * 32;
      // the choice bits of the thread's 32 columns (at most 4 groups of 8)
      // from one staged byte: S >= 8 and k0 a multiple of 32 keep them in it
      uint32_t cbyte = 0u;
      if (!sign_choice && rok && k0 < a.K) {
        const int bit0 = k0 >> a.ls;
        cbyte = (uint32_t)cbrow[(bit0 >> 3) - bb_lo] >> (bit0 & 7);
      }
      // the scale of the thread's first column: with g >= 32 it covers all 32
      uint32_t sraw0 = 0u;
      if (rok && k0 < a.K) {
        const int gl0 = (k0 >> a.lg) - gi_lo;
        sraw0 = FMT == kInt4 ? (uint32_t)reinterpret_cast<const unsigned short*>(scrow)[gl0]
                             : (uint32_t)scrow[gl0];
      }
      const bool one_scale = a.lg >= 5;
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int k = k0 + 8 * j;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (rok && k < a.K) {
          uint32_t tag, sraw = sraw0;
          if (!one_scale && j > 0) {
            const int gl = (k >> a.lg) - gi_lo;
            sraw = FMT == kInt4 ? (uint32_t)reinterpret_cast<const unsigned short*>(scrow)[gl]
                                : (uint32_t)scrow[gl];
          }
          const uint32_t cbit = (cbyte >> ((8 * j) >> a.ls)) & 1u;
          if (FMT == kNvfp4G) {
            tag = sraw >> 7;
            v = expand8g(words[j], __fmul_rn(gsv, e4m3_mag(sraw & 0x7fu)), sign_choice ? tag : cbit, sT);
          } else {
            const uint32_t sbf = scale_bits<FMT>(sraw, &tag);
            v = expand8(words[j], sbf, sign_choice ? tag : cbit, sT);
          }
        }
        const uint32_t c = (uint32_t)(h * 4 + j);
        *reinterpret_cast<uint4*>(dst + ((c ^ rsw) << 4)) = v;
      }
      fence_proxy_async();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[s]);
    }
    // the partial tile: TMEM lane quadrant of this warp = 32 weight rows
    const bool got = __all_sync(0xffffffffu, mbar_wait(accum, 0));
    tc_fence_after();
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const bool fail = !got || s_fail;
    constexpr int NC = BT / 2;
    uint32_t r[NC];
    if (!fail) tmem_ld_cols<NC>(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * NC), r);
    // all MMAs are complete (accum), so the A stages are free for the partials
#pragma unroll
    for (int j = 0; j < NC; j++)
      P[(half * NC + j) * kBN + q * 32 + lane] = fail ? __int_as_float(0x7fc00000) : __uint_as_float(r[j]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(small_tmem_cols<BT>()));
  }
  cluster_sync_all();  // every CTA's partial is in its shared memory
  {
    const int E = BT * kBN;
    const int e0 = (int)(crank * (uint32_t)E / csize), e1 = (int)((crank + 1) * (uint32_t)E / csize);
    for (int e = e0 + threadIdx.x; e < e1; e += kGemmThreads) {
      const int t = e / kBN, row = e % kBN;
      if (t < a.M && n0 + row < a.N) {
        float v = 0.0f;
        for (uint32_t c = 0; c < csize; c++) v = __fadd_rn(v, ld_cluster_f32(P + e, c));
        a.Y[(int64_t)t * a.N + n0 + row] = v;
      }
    }
  }
  cluster_sync_all();  // no CTA leaves while another may still read its partial
}

// ---------------------------------------------------------------------------
// host: tensor map for X through the driver entry point (no link to libcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cudaError_t encode_fn(EncodeTiledFn* out) {
  static std::mutex mu;
  static EncodeTiledFn fn = nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  *out = fn;
  return cudaSuccess;
}

template <int BT>
size_t gemm_smem() {
  return 1024 + (size_t)kStagesG * (kATileBytes + BT * 128) + (2 * kStagesG + 1) * 8 + 16;
}

template <int FMT, int BT>
cudaError_t launch_gemm_t(const uint16_t* X, int64_t M, int64_t ldx, const GemmArgs& ga,
                          cudaStream_t st) {
  EncodeTiledFn enc;
  cudaError_t e = encode_fn(&enc);
  if (e != cudaSuccess) return e;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)ga.K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BT};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const size_t smem = gemm_smem<BT>();
  e = cudaFuncSetAttribute(gemm_kernel<FMT, BT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned nblk = (unsigned)((ga.N + kBN - 1) / kBN), tblk = (unsigned)((M + BT - 1) / BT);
  GemmArgs g2 = ga;
  // fewer tiles than SMs: split K in two (the second half may be empty for K <= 64)
  g2.split = ((int64_t)nblk * tblk < 148 && ga.K > kBK) ? 2 : 1;
  if (g2.split == 2) {
    e = cudaMemsetAsync(ga.Y, 0, (size_t)M * (size_t)ga.N * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(nblk, tblk, (unsigned)g2.split);
  gemm_kernel<FMT, BT><<<grid, kGemmThreads, smem, st>>>(map, g2);
  return cudaGetLastError();
}

size_t gemm_tma_smem() {
  return 1024 + (size_t)kStagesT * (kATileBytes + kBTT * 128) + (2 * kStagesT + 4) * 8 + 16;
}

cudaError_t launch_gemm_tma(const uint16_t* X, int64_t M, int64_t ldx, const uint16_t* Wh,
                            const GemmArgs& ga, cudaStream_t st) {
  EncodeTiledFn enc;
  cudaError_t e = encode_fn(&enc);
  if (e != cudaSuccess) return e;
  CUtensorMap xmap, wmap;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)ga.K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBTT};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)ga.K, (cuuint64_t)ga.N};
    const cuuint64_t strides[1] = {(cuuint64_t)ga.K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBN};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(Wh), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = gemm_tma_smem();
  e = cudaFuncSetAttribute(gemm_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles_n = (int)((ga.N + kBN - 1) / kBN), tiles_t = (int)((M + kBTT - 1) / kBTT);
  const int tiles = tiles_n * tiles_t;
  const int grid = tiles < 148 ? tiles : 148;
  gemm_tma_kernel<<<grid, kGemmThreads, smem, st>>>(xmap, wmap, ga, tiles_t, tiles);
  return cudaGetLastError();
}

template <int BT>
size_t small_smem(int sc_stride, int cb_stride) {
  return 1024 + (size_t)kStagesS * (kATileBytes + BT * 128 + kCodeTileBytes) +
         (size_t)kBN * (sc_stride + cb_stride) + 8 + (3 * kStagesS + 1) * 8 + 16;
}

// Cluster size: about 240 CTAs over the layer's 128-row tiles, at least 2 and
// at most 8 (and no more than the K blocks).  Measured at 16 tokens (us):
// gate_proj 14336x4096 (112 tiles): C = 1 56, 2 43, 4 47, 8 55; q_proj
// 4096x4096 (32 tiles): C = 2 32.8, 4 22.6, 8 21.3; down_proj 4096x14336:
// 86.9, 51.1, 39.6; k_proj 1024x4096 (8 tiles): 32.6, 21.3, 17.1.  Fewer CTAs
// leave SMs idle; more, shorter ones spend more of their time filling and
// draining their stage rings.
int small_cluster(int tiles, int nkb) {
  int c = (240 + tiles / 2) / tiles;
  c = c < 2 ? 2 : (c > 8 ? 8 : c);
  return c < nkb ? c : nkb;
}

// Per-row staging of the largest CTA's scales and choice bytes (+2 for a
// range that straddles group and byte boundaries), rounded to 4 bytes.
void small_strides(int tiles, int nkb_all, int fmt, int lg, int ls, int* sc_stride,
                   int* cb_stride) {
  const int C = small_cluster(tiles, nkb_all);
  const int nkb_max = (nkb_all + C - 1) / C;
  const int esz = fmt == kInt4 ? 2 : 1;
  const int ng_max = (nkb_max * kBK) / (1 << lg) + 2;
  *sc_stride = (ng_max * esz + 3) & ~3;
  const int nbb_max = (nkb_max * kBK / (1 << ls)) / 8 + 2;
  *cb_stride = lg == ls ? 0 : ((nbb_max + 3) & ~3);
}

template <int FMT, int BT>
cudaError_t launch_gemm_small_t(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                                SmallArgs sa, cudaStream_t st) {
  EncodeTiledFn enc;
  cudaError_t e = encode_fn(&enc);
  if (e != cudaSuccess) return e;
  CUtensorMap xmap, cmap;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)sa.K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BT};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // codes as bytes: K / 2 per row (a multiple of 16: K % 32 == 0 is checked
    // by the caller); rows past N and bytes past K / 2 read as zero
    const cuuint64_t dims[2] = {(cuuint64_t)(sa.K / 2), (cuuint64_t)sa.N};
    const cuuint64_t strides[1] = {(cuuint64_t)(sa.K / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)(kBK / 2), (cuuint32_t)kBN};
    if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int tiles = (int)((sa.N + kBN - 1) / kBN);
  const int C = small_cluster(tiles, sa.nkb_all);
  small_strides(tiles, sa.nkb_all, FMT, sa.lg, sa.ls, &sa.sc_stride, &sa.cb_stride);
  const size_t smem = small_smem<BT>(sa.sc_stride, sa.cb_stride);
  if (smem > (size_t)kSmallSmemMax) return cudaErrorInvalidValue;  // gemm_small_fits checks it
  e = cudaFuncSetAttribute(gemm_small_kernel<FMT, BT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles, (unsigned)C, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)C;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_small_kernel<FMT, BT>, xmap, cmap, sa);
}

template <int FMT>
cudaError_t launch_gemm_small_f(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                                const SmallArgs& sa, cudaStream_t st) {
  if (M <= 16) return launch_gemm_small_t<FMT, 16>(X, M, ldx, codes, sa, st);
  return launch_gemm_small_t<FMT, 32>(X, M, ldx, codes, sa, st);
}

}  // namespace

cudaError_t launch_gemm(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                        const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                        int64_t K, int fmt, int lg, int ls, float* Y, const float* gsc,
                        cudaStream_t st) {
  GemmArgs ga{codes, tagged, cbits, Tb, Y, (int)M, (int)N, (int)K, lg, ls, 1, gsc};
  // token tile: 64 up to 64 tokens, then 128 (two CTAs fit on an SM), and 256
  // once there are at least two such tiles (less re-expansion of W per token)
  const int bt = M <= 64 ? 64 : (M < 512 ? 128 : 256);
  if (fmt == kInt4) {
    return bt == 64 ? launch_gemm_t<kInt4, 64>(X, M, ldx, ga, st)
         : bt == 128 ? launch_gemm_t<kInt4, 128>(X, M, ldx, ga, st)
                     : launch_gemm_t<kInt4, 256>(X, M, ldx, ga, st);
  }
  if (fmt == kNvfp4) {
    return bt == 64 ? launch_gemm_t<kNvfp4, 64>(X, M, ldx, ga, st)
         : bt == 128 ? launch_gemm_t<kNvfp4, 128>(X, M, ldx, ga, st)
                     : launch_gemm_t<kNvfp4, 256>(X, M, ldx, ga, st);
  }
  return bt == 64 ? launch_gemm_t<kNvfp4G, 64>(X, M, ldx, ga, st)
       : bt == 128 ? launch_gemm_t<kNvfp4G, 128>(X, M, ldx, ga, st)
                   : launch_gemm_t<kNvfp4G, 256>(X, M, ldx, ga, st);
}

bool gemm_small_fits(int64_t M, int64_t N, int64_t K, int fmt, int lg, int ls) {
  if (M < kSmallMinM || M > kSmallMaxM || K % 32 != 0) return false;
  // the staged scales and choice bytes grow with K: past the shared-memory
  // limit the fused kernel takes the layer
  int sc = 0, cb = 0;
  small_strides((int)((N + kBN - 1) / kBN), (int)((K + kBK - 1) / kBK), fmt, lg, ls, &sc, &cb);
  return small_smem<32>(sc, cb) <= (size_t)kSmallSmemMax;
}

void small_linear_plan(int64_t N, int64_t K, int fmt, int lg, int ls, int32_t* out) {
  const int nkb = (int)((K + kBK - 1) / kBK);
  const int tiles = (int)((N + kBN - 1) / kBN);
  int sc = 0, cb = 0;
  small_strides(tiles, nkb, fmt, lg, ls, &sc, &cb);
  out[0] = small_cluster(tiles, nkb);
  out[1] = nkb;
  out[2] = sc;
  out[3] = cb;
  out[4] = (int32_t)small_smem<16>(sc, cb);
  out[5] = (int32_t)small_smem<32>(sc, cb);
  out[6] = kSmallSmemMax;
}

cudaError_t launch_gemm_small(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                              const void* tagged, const uint8_t* cbits, const uint16_t* Tb,
                              int64_t N, int64_t K, int fmt, int lg, int ls, float* Y,
                              const float* gsc, cudaStream_t st) {
  SmallArgs sa{tagged, cbits, Tb, Y, (int)M, (int)N, (int)K, lg, ls,
               (int)((K + kBK - 1) / kBK), 0, 0, gsc};
  if (fmt == kInt4) return launch_gemm_small_f<kInt4>(X, M, ldx, codes, sa, st);
  if (fmt == kNvfp4) return launch_gemm_small_f<kNvfp4>(X, M, ldx, codes, sa, st);
  return launch_gemm_small_f<kNvfp4G>(X, M, ldx, codes, sa, st);
}

cudaError_t launch_gemm_dequantised(const uint16_t* X, int64_t M, int64_t ldx,
                                    const uint16_t* Wh, int64_t N, int64_t K, float* Y,
                                    cudaStream_t st) {
  const GemmArgs ga{nullptr, nullptr, nullptr, nullptr, Y, (int)M, (int)N, (int)K, 0, 0, 1,
                     nullptr};
  return launch_gemm_tma(X, M, ldx, Wh, ga, st);
}

cudaError_t gemm_timeout_flag(unsigned int* out) {
  return cudaMemcpyFromSymbol(out, g_gemm_timeout, sizeof(unsigned int));
}

}  // namespace aaac
