// internal.h -- host-side launchers and workspace layout shared by the
// translation units of libaaac.so.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "aaac.h"

namespace aaac {

// ---- workspace sections (byte offsets, each 256-aligned) -----------------
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct ImportancePlan {
  int ncb;        // column strips (seg_cols wide)
  int rb;         // row blocks
  int64_t rows_per_rb;
  size_t partial_bytes;  // double [rb][K]
  size_t list_bytes;     // int32 [K] flagged columns + counter
  size_t total;
};
ImportancePlan plan_importance(int64_t T, int64_t K);

struct PassPlan {
  int ncb;        // column strips (seg_cols wide)
  int nrc;        // row chunks
  int rows_per_chunk;
  int blocks;     // ncb * nrc
};
PassPlan plan_pass(int64_t N, int64_t K, int target_blocks = 148 * 4, int seg_cols = 256);

size_t fit_ctl_bytes();
size_t init_ctl_bytes();
size_t pack_extra_bytes(int64_t N, int64_t K, int S);
// the fit's workspace: control block + the (s, 1/s_eff) pair of every scale group
size_t fit_ws_bytes(int64_t N, int64_t K, int g);
// the fit/pack launch plan: blocks, strips, items per strip, rows per item,
// items per warp
void fit_launch_plan(int64_t N, int64_t K, int64_t M_total, uint32_t flags, int32_t out[5]);

// ---- the fit's library-owned scratch (fit.cu) -----------------------------
size_t fixed_scratch_bytes();
cudaError_t fixed_scratch_ptr(void** out);

// ---- launch accounting (aaac_kernel_launches) ------------------------------
void count_launches(int n);

// ---- launchers (return cudaGetLastError() of their launches) --------------
cudaError_t launch_importance(const uint16_t* X, int64_t T, int64_t K, int64_t ldx, uint32_t flags,
                              float* I, void* ws, cudaStream_t st);
// gs_out / gsc: the per-tensor scale of AAAC_NVFP4_GS (device fp32 [1]);
// ignored for the other formats.
cudaError_t launch_init(const uint16_t* W, int64_t N, int64_t K, int fmt, int g, void* scales,
                        float* T, void* ws, float* gs_out, cudaStream_t st);
// rsc: N * K/g float2 of workspace for the scale pairs of fit_round (NULL:
// the rounds run fit_pass, with only the control block in ws)
cudaError_t launch_fit(const uint16_t* W, int64_t N, int64_t K, const float* I,
                       const void* scales, int fmt, int g, int S, int iters, uint32_t flags,
                       float* T, double* err_hist, aaac_stats* stats, void* ws, float2* rsc,
                       const float* gsc, cudaStream_t st);
cudaError_t launch_pack(const uint16_t* W, int64_t N, int64_t K, const float* I,
                        const void* scales, int fmt, int g, int S, uint32_t flags, const float* T,
                        uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                        uint8_t* choice_bits, double* err_final, void* ws, const float* gsc,
                        cudaStream_t st);

// ---- row-sharded fit: the caller's reduction over the shards ----------------
// fn enqueues an in-place reduction of `count` elements at the device address
// buf on `stream` (op: AAAC_REDUCE_SUM_I64, AAAC_REDUCE_MAX_I64,
// AAAC_REDUCE_SUM_I32, AAAC_REDUCE_MAX_I32) and returns 0 on success.
struct Reducer {
  aaac_reduce_fn fn;
  void* user;
  bool failed;
  bool run(void* buf, int64_t count, int op, cudaStream_t st) {
    if (failed) return false;
    if (fn(user, buf, count, op, (void*)st) != 0) failed = true;
    return !failed;
  }
};
cudaError_t launch_init_sharded(const uint16_t* W, int64_t N, int64_t K, int64_t M_total, int fmt,
                                int g, void* scales, float* T, void* ws, float* gs_out,
                                Reducer& red, cudaStream_t st);
cudaError_t launch_fit_sharded(const uint16_t* W, int64_t N, int64_t K, int64_t M_total,
                               const float* I, const void* scales, int fmt, int g, int S,
                               int iters, uint32_t flags, float* T, double* err_hist,
                               aaac_stats* stats, void* ws, const float* gsc, Reducer& red,
                               cudaStream_t st);
cudaError_t launch_pack_sharded(const uint16_t* W, int64_t N, int64_t K, int64_t M_total,
                                const float* I, const void* scales, int fmt, int g, int S,
                                uint32_t flags, const float* T, uint16_t* T_bf16, uint8_t* codes,
                                void* scales_tagged, uint8_t* choice_bits, double* err_final,
                                void* ws, const float* gsc, Reducer& red, cudaStream_t st);

cudaError_t launch_dequant(const uint8_t* codes, const void* tagged, const uint8_t* cbits,
                           const uint16_t* Tb, int64_t N, int64_t K, int fmt, int g, int S,
                           uint16_t* W_hat, const float* gsc, cudaStream_t st);
cudaError_t launch_linear(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                          const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                          int64_t K, int fmt, int g, int S, float* Y, const float* gsc,
                          cudaStream_t st);

cudaError_t launch_gemm(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                        const void* tagged, const uint8_t* cbits, const uint16_t* Tb, int64_t N,
                        int64_t K, int fmt, int lg, int ls, float* Y, const float* gsc,
                        cudaStream_t st);
// Y = X W_hat^T from an already dequantised bf16 W_hat [N][K] (both operands by TMA)
// W4A16 linear for 5 to 32 tokens (K % 32 == 0): one 128-row tile per
// cluster of 2 to 8 CTAs splitting K, codes and X by TMA, the two partials summed
// in rank order over distributed shared memory
constexpr int64_t kSmallMinM = 5;
constexpr int64_t kSmallMaxM = 32;
bool gemm_small_fits(int64_t M, int64_t N, int64_t K, int fmt, int lg, int ls);
// the cluster kernel's plan for a layer of N x K: out[0] cluster size,
// [1] 64-column K blocks, [2] / [3] staged bytes per row for scales / choice
// bits, [4] / [5] shared memory of the 16- / 32-token kernel, [6] its limit
void small_linear_plan(int64_t N, int64_t K, int fmt, int lg, int ls, int32_t* out);
// which kernel aaac_linear runs for M tokens: 0 GEMV, 1 cluster, 2 fused
int linear_path(int64_t M, int64_t N, int64_t K, int fmt, int g, int S);
cudaError_t launch_gemm_small(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* codes,
                              const void* tagged, const uint8_t* cbits, const uint16_t* Tb,
                              int64_t N, int64_t K, int fmt, int lg, int ls, float* Y,
                              const float* gsc, cudaStream_t st);
cudaError_t launch_gemm_dequantised(const uint16_t* X, int64_t M, int64_t ldx,
                                    const uint16_t* Wh, int64_t N, int64_t K, float* Y,
                                    cudaStream_t st);
cudaError_t gemm_timeout_flag(unsigned int* out);
// the first failed device-side check of a checked build in the fit and the
// init kernels (0: none, or not a checked build)
cudaError_t fit_check_flag(unsigned int* out);
cudaError_t init_check_flag(unsigned int* out);

cudaError_t launch_awq_prescale(const uint16_t* W, int64_t N, int64_t K, const float* I,
                                int64_t tokens, int j, float* c, float* Is, uint16_t* Wout,
                                cudaStream_t st);
cudaError_t launch_awq_keep(int j, const double* err_alpha, const void* const* src,
                            void* const* dst, const size_t* bytes, int segs, double* err_final,
                            int32_t* best, cudaStream_t st);

}  // namespace aaac
