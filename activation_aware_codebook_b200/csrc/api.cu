// api.cu -- the extern "C" entry points of libaaac.so (declared in aaac.h):
// argument validation on the host, workspace carving, and kernel launches.
// No call allocates memory; every check runs before the first launch, so an
// invalid call leaves all outputs untouched.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace aaac {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
}  // namespace aaac

namespace {

thread_local std::string g_last_error;

aaac_status fail(aaac_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

aaac_status ok() {
  g_last_error.clear();
  return AAAC_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

aaac_status check_cfg(const aaac_config* cfg) {
  if (!cfg) return fail(AAAC_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->fmt != AAAC_INT4 && cfg->fmt != AAAC_NVFP4 && cfg->fmt != AAAC_NVFP4_GS)
    return fail(AAAC_ERR_UNSUPPORTED, "fmt %d is not AAAC_INT4, AAAC_NVFP4 or AAAC_NVFP4_GS",
                cfg->fmt);
  if (cfg->fmt != AAAC_INT4 && cfg->g != 16)
    return fail(AAAC_ERR_UNSUPPORTED, "NVFP4 needs g == 16 (got %d)", cfg->g);
  if (cfg->fmt == AAAC_NVFP4_GS) {
    if (!cfg->global_scale)
      return fail(AAAC_ERR_INVALID_ARG, "AAAC_NVFP4_GS needs cfg->global_scale");
    if (reinterpret_cast<uintptr_t>(cfg->global_scale) & 3u)
      return fail(AAAC_ERR_ALIGN, "cfg->global_scale is not 4-byte aligned");
  }
  if (!pow2(cfg->g) || cfg->g < 16 || cfg->g > 256)
    return fail(AAAC_ERR_UNSUPPORTED, "g must be a power of two in [16, 256] (got %d)", cfg->g);
  if (!pow2(cfg->S) || cfg->S < 8 || cfg->S > cfg->g)
    return fail(AAAC_ERR_SHAPE, "S must be a power of two with 8 <= S <= g (S=%d, g=%d)",
                cfg->S, cfg->g);
  if (cfg->iters < 0) return fail(AAAC_ERR_INVALID_ARG, "iters < 0 (%d)", cfg->iters);
  if (cfg->flags & ~15u) return fail(AAAC_ERR_INVALID_ARG, "unknown flags 0x%x", cfg->flags);
  return AAAC_OK;
}

aaac_status check_layer(int64_t N, int64_t K, const aaac_config* cfg) {
  if (N <= 0 || K <= 0) return fail(AAAC_ERR_SHAPE, "N and K must be positive (N=%lld K=%lld)",
                                    (long long)N, (long long)K);
  if (K % cfg->g) return fail(AAAC_ERR_SHAPE, "K=%lld is not a multiple of g=%d", (long long)K,
                              cfg->g);
  if (N > INT32_MAX || K > INT32_MAX || N * K >= ((int64_t)1 << 31))
    return fail(AAAC_ERR_SHAPE, "N*K must be < 2^31 (N=%lld K=%lld)", (long long)N,
                (long long)K);
  return AAAC_OK;
}

aaac_status check_ptr(const void* p, const char* name, bool required = true) {
  if (!p) return required ? fail(AAAC_ERR_INVALID_ARG, "%s is NULL", name) : AAAC_OK;
  if (!aligned16(p)) return fail(AAAC_ERR_ALIGN, "%s is not 16-byte aligned", name);
  return AAAC_OK;
}

aaac_status check_ws(void* ws, size_t have, size_t need) {
  if (!ws) return fail(AAAC_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (!aligned16(ws)) return fail(AAAC_ERR_ALIGN, "workspace is not 16-byte aligned");
  if (have < need) return fail(AAAC_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", have, need);
  return AAAC_OK;
}

// NVTX range around a call (named in profiler timelines; no cost without a tool).
struct CallScope {
  explicit CallScope(const char* name) { nvtxRangePushA(name); }
  ~CallScope() { nvtxRangePop(); }
  CallScope(const CallScope&) = delete;
  CallScope& operator=(const CallScope&) = delete;
};

// Host-side fault injection, for tests of callers' error paths: one fault is
// armed by AAAC_FAULT=alloc|launch|sync in the environment when the library
// first runs a call, or by aaac_inject_fault().  The next call that would
// launch work then returns the matching status after its argument checks,
// before anything reaches the GPU, and leaves every output untouched.
enum { kFaultNone = 0, kFaultAlloc = 1, kFaultLaunch = 2, kFaultSync = 3 };
std::atomic<int> g_fault{kFaultNone};
std::once_flag g_fault_env;

int fault_kind(const char* k) {
  if (!k || !*k) return kFaultNone;
  if (!strcmp(k, "alloc")) return kFaultAlloc;
  if (!strcmp(k, "launch")) return kFaultLaunch;
  if (!strcmp(k, "sync")) return kFaultSync;
  return -1;
}

aaac_status take_fault() {
  std::call_once(g_fault_env, [] {
    const int k = fault_kind(getenv("AAAC_FAULT"));
    if (k > 0) g_fault.store(k);
  });
  switch (g_fault.exchange(kFaultNone)) {
    case kFaultAlloc:
      return fail(AAAC_ERR_WORKSPACE, "injected fault: workspace allocation failed");
    case kFaultLaunch:
      return fail(AAAC_ERR_CUDA, "injected fault: kernel launch failed");
    case kFaultSync:
      return fail(AAAC_ERR_CUDA, "injected fault: stream synchronisation failed");
    default:
      return AAAC_OK;
  }
}

aaac_status from_cuda(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return ok();
  return fail(AAAC_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

size_t weight_side_bytes(const aaac_config* cfg, int64_t N, int64_t K) {
  if (!cfg || N <= 0 || K <= 0 || cfg->S <= 0) return 0;
  size_t fit = aaac::fit_ws_bytes(N, K, cfg->g);
  size_t pack = aaac::fit_ctl_bytes() + aaac::pack_extra_bytes(N, K, cfg->S);
  size_t init = aaac::init_ctl_bytes();
  size_t m = fit > pack ? fit : pack;
  return m > init ? m : init;
}

// Workspace of aaac_awq_fit: the rescaled layer, one candidate's fit state
// and packed output, and the fit's own workspace (shared by init, fit, pack).
struct AwqLayout {
  size_t Ws, Is, c, scales, T, Tb, codes, tagged, bits, hist, stats, gs, fit, total;
};
AwqLayout awq_layout(const aaac_config* cfg, int64_t N, int64_t K) {
  AwqLayout L{};
  const int64_t G = K / cfg->g;
  const size_t es = cfg->fmt == AAAC_INT4 ? 2 : 1;
  const size_t nb = cfg->S != cfg->g ? (size_t)((K / cfg->S + 7) / 8) : 0;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += aaac::align256(bytes);
    return at;
  };
  L.Ws = take((size_t)(N * K) * 2);
  L.Is = take((size_t)K * 4);
  L.c = take((size_t)K * 4);
  L.scales = take((size_t)(N * G) * es);
  L.T = take(2 * 16 * 4);
  L.Tb = take(2 * 16 * 2);
  L.codes = take((size_t)(N * K / 2));
  L.tagged = take((size_t)(N * G) * es);
  L.bits = take((size_t)N * nb);
  L.hist = take((size_t)(cfg->iters > 0 ? cfg->iters : 1) * 8);
  L.stats = take(sizeof(aaac_stats));
  L.gs = take(sizeof(float));
  L.fit = take(weight_side_bytes(cfg, N, K));
  L.total = o;
  return L;
}

#define CHECK(x)                         \
  do {                                   \
    aaac_status _s = (x);                \
    if (_s != AAAC_OK) return _s;        \
  } while (0)

}  // namespace

extern "C" {

const char* aaac_last_error(void) { return g_last_error.c_str(); }

const char* aaac_version(void) { return "libaaac 0.1 (sm_100a)"; }

uint64_t aaac_kernel_launches(void) { return aaac::g_launches.load(std::memory_order_relaxed); }

aaac_status aaac_fit_launch_plan(const aaac_config* cfg, int64_t N, int64_t K, int64_t N_total,
                                 int32_t* out) {
  if (!out) return fail(AAAC_ERR_INVALID_ARG, "out is NULL");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  if (N_total < N)
    return fail(AAAC_ERR_SHAPE, "N_total=%lld < N=%lld", (long long)N_total, (long long)N);
  CHECK(check_layer(N_total, K, cfg));
  aaac::fit_launch_plan(N, K, N_total * K, cfg->flags, out);
  return ok();
}

aaac_status aaac_linear_launch_plan(const aaac_config* cfg, int64_t M, int64_t N, int64_t K,
                                    int32_t* out) {
  if (!out) return fail(AAAC_ERR_INVALID_ARG, "out is NULL");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  if (M < 1 || M > ((int64_t)1 << 20))
    return fail(AAAC_ERR_SHAPE, "M=%lld must be in [1, 2^20]", (long long)M);
  int lg = 0, ls = 0;
  while ((1 << lg) < cfg->g) lg++;
  while ((1 << ls) < cfg->S) ls++;
  out[0] = aaac::linear_path(M, N, K, cfg->fmt, cfg->g, cfg->S);
  aaac::small_linear_plan(N, K, cfg->fmt, lg, ls, out + 1);
  return ok();
}

size_t aaac_workspace_size(const aaac_config* cfg, int64_t N, int64_t K, int64_t T) {
  size_t need = weight_side_bytes(cfg, N, K);
  if (T > 0 && K > 0) {
    size_t imp = aaac::plan_importance(T, K).total;
    if (imp > need) need = imp;
  }
  return need < 256 ? 256 : need;
}

aaac_status aaac_importance(const void* X, int64_t T, int64_t K, int64_t ldx, uint32_t flags,
                            float* I, void* ws, size_t ws_bytes, void* stream) {
  CallScope cs_("aaac_importance");
  CHECK(check_ptr(X, "X"));
  CHECK(check_ptr(I, "I"));
  if (T <= 0 || K <= 0) return fail(AAAC_ERR_SHAPE, "T and K must be positive");
  if (K % 8 || ldx % 8) return fail(AAAC_ERR_ALIGN, "K and ldx must be multiples of 8");
  if (ldx < K) return fail(AAAC_ERR_SHAPE, "ldx (%lld) < K (%lld)", (long long)ldx, (long long)K);
  if (K > INT32_MAX || T > ((int64_t)1 << 40))
    return fail(AAAC_ERR_SHAPE, "K or T out of range");
  if (flags & ~3u) return fail(AAAC_ERR_INVALID_ARG, "unknown importance flags 0x%x", flags);
  CHECK(check_ws(ws, ws_bytes, aaac::plan_importance(T, K).total));
  CHECK(take_fault());
  return from_cuda(aaac::launch_importance(reinterpret_cast<const uint16_t*>(X), T, K, ldx, flags,
                                           I, ws, (cudaStream_t)stream),
                   "aaac_importance");
}

aaac_status aaac_init_codebooks(const void* W, int64_t N, int64_t K, const aaac_config* cfg,
                                void* scales, float* T, void* ws, size_t ws_bytes,
                                void* stream) {
  CallScope cs_("aaac_init_codebooks");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(scales, "scales"));
  CHECK(check_ptr(T, "T"));
  CHECK(check_ws(ws, ws_bytes, aaac::init_ctl_bytes()));
  CHECK(take_fault());
  return from_cuda(aaac::launch_init(reinterpret_cast<const uint16_t*>(W), N, K, cfg->fmt, cfg->g,
                                     scales, T, ws, cfg->global_scale, (cudaStream_t)stream),
                   "aaac_init_codebooks");
}

aaac_status aaac_fit_layer(const void* W, int64_t N, int64_t K, const float* I,
                           const void* scales, const aaac_config* cfg, float* T,
                           double* err_hist, aaac_stats* stats, void* ws, size_t ws_bytes,
                           void* stream) {
  CallScope cs_("aaac_fit_layer");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(I, "I"));
  CHECK(check_ptr(scales, "scales"));
  CHECK(check_ptr(T, "T"));
  CHECK(check_ptr(err_hist, "err_hist", false));
  CHECK(check_ptr(stats, "stats", false));
  CHECK(check_ws(ws, ws_bytes, aaac::fit_ws_bytes(N, K, cfg->g)));
  float2* rsc = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(ws) + aaac::fit_ctl_bytes());
  CHECK(take_fault());
  return from_cuda(aaac::launch_fit(reinterpret_cast<const uint16_t*>(W), N, K, I, scales,
                                    cfg->fmt, cfg->g, cfg->S, cfg->iters, cfg->flags, T, err_hist,
                                    stats, ws, rsc, cfg->global_scale, (cudaStream_t)stream),
                   "aaac_fit_layer");
}

aaac_status aaac_fit_layer_fixed_scratch(const void* W, int64_t N, int64_t K, const float* I,
                                         const void* scales, const aaac_config* cfg, float* T,
                                         double* err_hist, aaac_stats* stats, void* stream) {
  CallScope cs_("aaac_fit_layer_fixed_scratch");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(I, "I"));
  CHECK(check_ptr(scales, "scales"));
  CHECK(check_ptr(T, "T"));
  CHECK(check_ptr(err_hist, "err_hist", false));
  CHECK(check_ptr(stats, "stats", false));
  // with no room for per-layer tables the rounds run fit_pass, whose only
  // scratch is the control block
  const size_t need = aaac::fit_ctl_bytes();
  if (need > aaac::fixed_scratch_bytes())
    return fail(AAAC_ERR_WORKSPACE,
                "this layer (N=%lld K=%lld) needs %zu bytes of scratch but the library's fixed "
                "scratch holds %zu; call aaac_fit_layer with a workspace instead",
                (long long)N, (long long)K, need, aaac::fixed_scratch_bytes());
  void* ws = nullptr;
  CHECK(take_fault());
  cudaError_t e = aaac::fixed_scratch_ptr(&ws);
  if (e != cudaSuccess) return from_cuda(e, "aaac_fit_layer_fixed_scratch: scratch address");
  return from_cuda(aaac::launch_fit(reinterpret_cast<const uint16_t*>(W), N, K, I, scales,
                                    cfg->fmt, cfg->g, cfg->S, cfg->iters, cfg->flags, T, err_hist,
                                    stats, ws, nullptr, cfg->global_scale, (cudaStream_t)stream),
                   "aaac_fit_layer_fixed_scratch");
}

aaac_status aaac_pack(const void* W, int64_t N, int64_t K, const float* I, const void* scales,
                      const aaac_config* cfg, const float* T, uint16_t* T_bf16, uint8_t* codes,
                      void* scales_tagged, uint8_t* choice_bits, double* err_final, void* ws,
                      size_t ws_bytes, void* stream) {
  CallScope cs_("aaac_pack");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(I, "I"));
  CHECK(check_ptr(scales, "scales"));
  CHECK(check_ptr(T, "T"));
  CHECK(check_ptr(T_bf16, "T_bf16"));
  CHECK(check_ptr(codes, "codes"));
  CHECK(check_ptr(scales_tagged, "scales_tagged"));
  CHECK(check_ptr(choice_bits, "choice_bits", cfg->S != cfg->g));
  CHECK(check_ptr(err_final, "err_final", false));
  CHECK(check_ws(ws, ws_bytes, aaac::fit_ctl_bytes() + aaac::pack_extra_bytes(N, K, cfg->S)));
  CHECK(take_fault());
  return from_cuda(aaac::launch_pack(reinterpret_cast<const uint16_t*>(W), N, K, I, scales,
                                     cfg->fmt, cfg->g, cfg->S, cfg->flags, T, T_bf16, codes,
                                     scales_tagged, choice_bits, err_final, ws, cfg->global_scale,
                                     (cudaStream_t)stream),
                   "aaac_pack");
}

aaac_status aaac_dequant(const uint8_t* codes, const void* scales_tagged,
                         const uint8_t* choice_bits, const uint16_t* T_bf16, int64_t N, int64_t K,
                         const aaac_config* cfg, uint16_t* W_hat, void* stream) {
  CallScope cs_("aaac_dequant");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_ptr(codes, "codes"));
  CHECK(check_ptr(scales_tagged, "scales_tagged"));
  CHECK(check_ptr(choice_bits, "choice_bits", cfg->S != cfg->g));
  CHECK(check_ptr(T_bf16, "T_bf16"));
  CHECK(check_ptr(W_hat, "W_hat"));
  CHECK(take_fault());
  return from_cuda(aaac::launch_dequant(codes, scales_tagged, choice_bits, T_bf16, N, K, cfg->fmt,
                                        cfg->g, cfg->S, W_hat, cfg->global_scale,
                                        (cudaStream_t)stream),
                   "aaac_dequant");
}

aaac_status aaac_linear(const void* X, int64_t M, int64_t ldx, const uint8_t* codes,
                        const void* scales_tagged, const uint8_t* choice_bits,
                        const uint16_t* T_bf16, int64_t N, int64_t K, const aaac_config* cfg,
                        float* Y, void* stream) {
  CallScope cs_("aaac_linear");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  if (M < 1 || M > ((int64_t)1 << 20))
    return fail(AAAC_ERR_SHAPE, "M=%lld must be in [1, 2^20]", (long long)M);
  if (ldx < K) return fail(AAAC_ERR_SHAPE, "ldx=%lld < K=%lld", (long long)ldx, (long long)K);
  if (ldx % 8) return fail(AAAC_ERR_ALIGN, "ldx=%lld is not a multiple of 8", (long long)ldx);
  if (M * ldx >= ((int64_t)1 << 40))
    return fail(AAAC_ERR_SHAPE, "M*ldx is too large (M=%lld ldx=%lld)", (long long)M,
                (long long)ldx);
  CHECK(check_ptr(X, "X"));
  CHECK(check_ptr(codes, "codes"));
  CHECK(check_ptr(scales_tagged, "scales_tagged"));
  CHECK(check_ptr(choice_bits, "choice_bits", cfg->S != cfg->g));
  CHECK(check_ptr(T_bf16, "T_bf16"));
  CHECK(check_ptr(Y, "Y"));
  CHECK(take_fault());
  return from_cuda(aaac::launch_linear(reinterpret_cast<const uint16_t*>(X), M, ldx, codes,
                                       scales_tagged, choice_bits, T_bf16, N, K, cfg->fmt,
                                       cfg->g, cfg->S, Y, cfg->global_scale, (cudaStream_t)stream),
                   "aaac_linear");
}

aaac_status aaac_awq_prescale(const void* W, int64_t N, int64_t K, const float* I,
                              int64_t tokens, int alpha16, float* c, float* I_scaled,
                              void* W_scaled, void* stream) {
  CallScope cs_("aaac_awq_prescale");
  if (N <= 0 || K <= 0) return fail(AAAC_ERR_SHAPE, "N and K must be positive");
  if (K % 8) return fail(AAAC_ERR_ALIGN, "K=%lld is not a multiple of 8", (long long)K);
  if (N > INT32_MAX || K > INT32_MAX || N * K >= ((int64_t)1 << 31))
    return fail(AAAC_ERR_SHAPE, "N*K must be < 2^31 (N=%lld K=%lld)", (long long)N,
                (long long)K);
  if (tokens <= 0) return fail(AAAC_ERR_SHAPE, "tokens must be positive (%lld)", (long long)tokens);
  if (alpha16 < 0 || alpha16 > 16)
    return fail(AAAC_ERR_INVALID_ARG, "alpha16=%d is not in [0, 16]", alpha16);
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(I, "I"));
  CHECK(check_ptr(c, "c"));
  CHECK(check_ptr(I_scaled, "I_scaled"));
  CHECK(check_ptr(W_scaled, "W_scaled"));
  CHECK(take_fault());
  return from_cuda(aaac::launch_awq_prescale(reinterpret_cast<const uint16_t*>(W), N, K, I,
                                             tokens, alpha16, c, I_scaled,
                                             reinterpret_cast<uint16_t*>(W_scaled),
                                             (cudaStream_t)stream),
                   "aaac_awq_prescale");
}

size_t aaac_awq_workspace_size(const aaac_config* cfg, int64_t N, int64_t K) {
  if (!cfg || N <= 0 || K <= 0 || cfg->g <= 0 || cfg->S <= 0 || K % cfg->g) return 0;
  return awq_layout(cfg, N, K).total;
}

aaac_status aaac_awq_fit(const void* W, int64_t N, int64_t K, const float* I, int64_t tokens,
                         const aaac_config* cfg, const int32_t* alpha16, int n_alpha, float* c,
                         uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                         uint8_t* choice_bits, double* err_final, double* err_alpha,
                         int32_t* best, void* ws, size_t ws_bytes, void* stream) {
  CallScope cs_("aaac_awq_fit");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  if (tokens <= 0) return fail(AAAC_ERR_SHAPE, "tokens must be positive (%lld)", (long long)tokens);
  if (!alpha16) return fail(AAAC_ERR_INVALID_ARG, "alpha16 is NULL");
  if (n_alpha < 1 || n_alpha > 17)
    return fail(AAAC_ERR_INVALID_ARG, "n_alpha=%d is not in [1, 17]", n_alpha);
  for (int i = 0; i < n_alpha; i++)
    if (alpha16[i] < 0 || alpha16[i] > 16)
      return fail(AAAC_ERR_INVALID_ARG, "alpha16[%d]=%d is not in [0, 16]", i, alpha16[i]);
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(I, "I"));
  CHECK(check_ptr(c, "c"));
  CHECK(check_ptr(T_bf16, "T_bf16"));
  CHECK(check_ptr(codes, "codes"));
  CHECK(check_ptr(scales_tagged, "scales_tagged"));
  CHECK(check_ptr(choice_bits, "choice_bits", cfg->S != cfg->g));
  CHECK(check_ptr(err_final, "err_final", false));
  CHECK(check_ptr(err_alpha, "err_alpha"));
  CHECK(check_ptr(best, "best", false));
  const AwqLayout L = awq_layout(cfg, N, K);
  CHECK(check_ws(ws, ws_bytes, L.total));
  unsigned char* base = static_cast<unsigned char*>(ws);
  uint16_t* Ws = reinterpret_cast<uint16_t*>(base + L.Ws);
  float* Is = reinterpret_cast<float*>(base + L.Is);
  float* cc = reinterpret_cast<float*>(base + L.c);
  void* scl = base + L.scales;
  float* T = reinterpret_cast<float*>(base + L.T);
  uint16_t* Tb = reinterpret_cast<uint16_t*>(base + L.Tb);
  uint8_t* cod = base + L.codes;
  void* tag = base + L.tagged;
  uint8_t* bits = cfg->S != cfg->g ? base + L.bits : nullptr;
  double* hist = reinterpret_cast<double*>(base + L.hist);
  aaac_stats* stats = reinterpret_cast<aaac_stats*>(base + L.stats);
  void* fws = base + L.fit;
  // candidates keep their tensor scale (NVFP4_GS) in the workspace; the kept
  // one is copied to cfg->global_scale with the rest of its output
  float* gs = cfg->fmt == AAAC_NVFP4_GS ? reinterpret_cast<float*>(base + L.gs) : nullptr;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t G = K / cfg->g;
  const size_t es = cfg->fmt == AAAC_INT4 ? 2 : 1;
  const void* src[6] = {cod, tag, Tb, cc, bits, gs};
  void* dst[6] = {codes, scales_tagged, T_bf16, c, choice_bits, cfg->global_scale};
  const size_t bytes[6] = {(size_t)(N * K / 2), (size_t)(N * G) * es, 2 * 16 * 2, (size_t)K * 4,
                           bits ? (size_t)N * ((K / cfg->S + 7) / 8) : 0, gs ? sizeof(float) : 0};
  CHECK(take_fault());
  for (int i = 0; i < n_alpha; i++) {
    cudaError_t e = aaac::launch_awq_prescale(reinterpret_cast<const uint16_t*>(W), N, K, I,
                                              tokens, alpha16[i], cc, Is, Ws, st);
    if (e == cudaSuccess)
      e = aaac::launch_init(Ws, N, K, cfg->fmt, cfg->g, scl, T, fws, gs, st);
    if (e == cudaSuccess)
      e = aaac::launch_fit(Ws, N, K, Is, scl, cfg->fmt, cfg->g, cfg->S, cfg->iters, cfg->flags, T,
                           hist, stats, fws,
                           reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(fws) +
                                                     aaac::fit_ctl_bytes()),
                           gs, st);
    if (e == cudaSuccess)
      e = aaac::launch_pack(Ws, N, K, Is, scl, cfg->fmt, cfg->g, cfg->S, cfg->flags, T, Tb, cod,
                            tag, bits, err_alpha + i, fws, gs, st);
    if (e == cudaSuccess)
      e = aaac::launch_awq_keep(i, err_alpha, src, dst, bytes, 6, err_final, best, st);
    if (e != cudaSuccess) return from_cuda(e, "aaac_awq_fit");
  }
  return ok();
}

static aaac_status check_shards(int64_t N, int64_t K, int64_t N_total, const aaac_config* cfg,
                                aaac_reduce_fn reduce) {
  if (!reduce) return fail(AAAC_ERR_INVALID_ARG, "reduce is NULL");
  if (N_total < N)
    return fail(AAAC_ERR_SHAPE, "N_total=%lld < N=%lld", (long long)N_total, (long long)N);
  return check_layer(N_total, K, cfg);  // the whole layer obeys the unsharded limits
}

aaac_status aaac_init_codebooks_sharded(const void* W, int64_t N, int64_t K, int64_t N_total,
                                        const aaac_config* cfg, void* scales, float* T,
                                        aaac_reduce_fn reduce, void* user, void* ws,
                                        size_t ws_bytes, void* stream) {
  CallScope cs_("aaac_init_codebooks_sharded");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_shards(N, K, N_total, cfg, reduce));
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(scales, "scales"));
  CHECK(check_ptr(T, "T"));
  CHECK(check_ws(ws, ws_bytes, aaac::init_ctl_bytes()));
  CHECK(take_fault());
  aaac::Reducer red{reduce, user, false};
  const cudaError_t e = aaac::launch_init_sharded(reinterpret_cast<const uint16_t*>(W), N, K,
                                                  N_total * K, cfg->fmt, cfg->g, scales, T, ws,
                                                  cfg->global_scale, red, (cudaStream_t)stream);
  if (red.failed) return fail(AAAC_ERR_COLLECTIVE, "aaac_init_codebooks_sharded: reduce failed");
  return from_cuda(e, "aaac_init_codebooks_sharded");
}

aaac_status aaac_fit_layer_sharded(const void* W, int64_t N, int64_t K, int64_t N_total,
                                   const float* I, const void* scales, const aaac_config* cfg,
                                   float* T, double* err_hist, aaac_stats* stats,
                                   aaac_reduce_fn reduce, void* user, void* ws, size_t ws_bytes,
                                   void* stream) {
  CallScope cs_("aaac_fit_layer_sharded");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_shards(N, K, N_total, cfg, reduce));
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(I, "I"));
  CHECK(check_ptr(scales, "scales"));
  CHECK(check_ptr(T, "T"));
  CHECK(check_ptr(err_hist, "err_hist", false));
  CHECK(check_ptr(stats, "stats", false));
  CHECK(check_ws(ws, ws_bytes, aaac::fit_ws_bytes(N, K, cfg->g)));
  CHECK(take_fault());
  aaac::Reducer red{reduce, user, false};
  const cudaError_t e = aaac::launch_fit_sharded(
      reinterpret_cast<const uint16_t*>(W), N, K, N_total * K, I, scales, cfg->fmt, cfg->g,
      cfg->S, cfg->iters, cfg->flags, T, err_hist, stats, ws, cfg->global_scale, red,
      (cudaStream_t)stream);
  if (red.failed) return fail(AAAC_ERR_COLLECTIVE, "aaac_fit_layer_sharded: reduce failed");
  return from_cuda(e, "aaac_fit_layer_sharded");
}

aaac_status aaac_pack_sharded(const void* W, int64_t N, int64_t K, int64_t N_total,
                              const float* I, const void* scales, const aaac_config* cfg,
                              const float* T, uint16_t* T_bf16, uint8_t* codes,
                              void* scales_tagged, uint8_t* choice_bits, double* err_final,
                              aaac_reduce_fn reduce, void* user, void* ws, size_t ws_bytes,
                              void* stream) {
  CallScope cs_("aaac_pack_sharded");
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  CHECK(check_shards(N, K, N_total, cfg, reduce));
  CHECK(check_ptr(W, "W"));
  CHECK(check_ptr(I, "I"));
  CHECK(check_ptr(scales, "scales"));
  CHECK(check_ptr(T, "T"));
  CHECK(check_ptr(T_bf16, "T_bf16"));
  CHECK(check_ptr(codes, "codes"));
  CHECK(check_ptr(scales_tagged, "scales_tagged"));
  CHECK(check_ptr(choice_bits, "choice_bits", cfg->S != cfg->g));
  CHECK(check_ptr(err_final, "err_final", false));
  CHECK(check_ws(ws, ws_bytes, aaac::fit_ctl_bytes() + aaac::pack_extra_bytes(N, K, cfg->S)));
  CHECK(take_fault());
  aaac::Reducer red{reduce, user, false};
  const cudaError_t e = aaac::launch_pack_sharded(
      reinterpret_cast<const uint16_t*>(W), N, K, N_total * K, I, scales, cfg->fmt, cfg->g,
      cfg->S, cfg->flags, T, T_bf16, codes, scales_tagged, choice_bits, err_final, ws,
      cfg->global_scale, red, (cudaStream_t)stream);
  if (red.failed) return fail(AAAC_ERR_COLLECTIVE, "aaac_pack_sharded: reduce failed");
  return from_cuda(e, "aaac_pack_sharded");
}

// Token counts from which aaac_linear_ws dequantises W once into its
// workspace and runs the TMA-fed GEMM (below it the fused kernels are faster).
static const int64_t kDequantMinM = 192;

size_t aaac_linear_workspace_size(const aaac_config* cfg, int64_t M, int64_t N, int64_t K) {
  if (!cfg || M < kDequantMinM || N <= 0 || K <= 0) return 0;
  return aaac::align256((size_t)N * (size_t)K * 2);
}

aaac_status aaac_linear_ws(const void* X, int64_t M, int64_t ldx, const uint8_t* codes,
                           const void* scales_tagged, const uint8_t* choice_bits,
                           const uint16_t* T_bf16, int64_t N, int64_t K, const aaac_config* cfg,
                           float* Y, void* ws, size_t ws_bytes, void* stream) {
  CallScope cs_("aaac_linear_ws");
  const size_t need = aaac_linear_workspace_size(cfg, M, N, K);
  if (need == 0 || !ws || ws_bytes < need || !aligned16(ws))
    return aaac_linear(X, M, ldx, codes, scales_tagged, choice_bits, T_bf16, N, K, cfg, Y, stream);
  CHECK(check_cfg(cfg));
  CHECK(check_layer(N, K, cfg));
  if (M > ((int64_t)1 << 20))
    return fail(AAAC_ERR_SHAPE, "M=%lld must be in [1, 2^20]", (long long)M);
  if (ldx < K) return fail(AAAC_ERR_SHAPE, "ldx=%lld < K=%lld", (long long)ldx, (long long)K);
  if (ldx % 8) return fail(AAAC_ERR_ALIGN, "ldx=%lld is not a multiple of 8", (long long)ldx);
  if (M * ldx >= ((int64_t)1 << 40))
    return fail(AAAC_ERR_SHAPE, "M*ldx is too large (M=%lld ldx=%lld)", (long long)M,
                (long long)ldx);
  CHECK(check_ptr(X, "X"));
  CHECK(check_ptr(codes, "codes"));
  CHECK(check_ptr(scales_tagged, "scales_tagged"));
  CHECK(check_ptr(choice_bits, "choice_bits", cfg->S != cfg->g));
  CHECK(check_ptr(T_bf16, "T_bf16"));
  CHECK(check_ptr(Y, "Y"));
  uint16_t* Wh = static_cast<uint16_t*>(ws);
  CHECK(take_fault());
  cudaError_t e = aaac::launch_dequant(codes, scales_tagged, choice_bits, T_bf16, N, K, cfg->fmt,
                                       cfg->g, cfg->S, Wh, cfg->global_scale,
                                       (cudaStream_t)stream);
  if (e == cudaSuccess)
    e = aaac::launch_gemm_dequantised(reinterpret_cast<const uint16_t*>(X), M, ldx, Wh, N, K, Y,
                                      (cudaStream_t)stream);
  if (e == cudaSuccess) aaac::count_launches(1);
  return from_cuda(e, "aaac_linear_ws");
}

aaac_status aaac_device_checks(uint32_t* flag) {
  if (!flag) return fail(AAAC_ERR_INVALID_ARG, "flag is NULL");
  unsigned int vf = 0, vi = 0;
  cudaError_t e = aaac::fit_check_flag(&vf);
  if (e == cudaSuccess) e = aaac::init_check_flag(&vi);
  if (e != cudaSuccess) return from_cuda(e, "aaac_device_checks");
  *flag = vf ? vf : vi;
  return ok();
}

int aaac_checked_build(void) {
#ifdef AAAC_CHECKS
  return 1;
#else
  return 0;
#endif
}

aaac_status aaac_inject_fault(const char* kind) {
  const int k = fault_kind(kind);
  if (k < 0)
    return fail(AAAC_ERR_INVALID_ARG, "unknown fault kind '%s' (alloc, launch, sync or empty)",
                kind);
  g_fault.store(k);
  return ok();
}

aaac_status aaac_device_timeouts(uint32_t* flag) {
  if (!flag) return fail(AAAC_ERR_INVALID_ARG, "flag is NULL");
  unsigned int v = 0;
  const cudaError_t e = aaac::gemm_timeout_flag(&v);
  if (e != cudaSuccess) return from_cuda(e, "aaac_device_timeouts");
  *flag = v ? 1u : 0u;
  return AAAC_OK;
}

}  // extern "C"
