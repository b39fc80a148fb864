/*
 * aaac.h -- C ABI of libaaac.so, the B200 (sm_100a) implementation of the
 * per-layer codebook fit of AAAC (activation-aware adaptive codebooks) for
 * 4-bit group-scaled weights.
 *
 * Source of the method: "Technical summary: AAAC (activation-aware adaptive
 * codebooks)", gist.science/ko/paper/2605.08692.  Section references below
 * are to that page.
 *
 * Conventions shared by every call
 *  - All tensors are caller-allocated DEVICE memory on the current CUDA device,
 *    except the aaac_config struct, which is host memory read during the call.
 *    The library allocates nothing: scratch memory is the caller's workspace
 *    (ws, ws_bytes), sized by aaac_workspace_size().  The one exception is
 *    aaac_fit_layer_fixed_scratch, which uses an array inside the library.
 *  - W is the weight, row-major [N][K] bf16 (N output rows, K input columns);
 *    groups of g (scale) and S (codebook choice) weights run along K.
 *    X is the calibration activation, row-major [T][ldx] bf16 (T tokens).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Outputs are valid once that stream has synchronised.
 *  - Pointers must be 16-byte aligned; K and ldx must be multiples of 8.
 *  - On an invalid argument a call returns an error BEFORE launching anything
 *    and leaves every output untouched.  A CUDA launch error maps to
 *    AAAC_ERR_CUDA.  aaac_last_error() gives a message for the calling thread.
 *  - Calls on one stream may share a workspace; concurrent calls on different
 *    streams need different workspaces.
 *  - NaN or infinite weights / activations are outside the contract: results
 *    are then unspecified, but every memory access stays in bounds.
 */
#ifndef AAAC_H
#define AAAC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AAAC_OK = 0,
    AAAC_ERR_INVALID_ARG = 1, /* null pointer, bad flag, iters < 0            */
    AAAC_ERR_SHAPE = 2,       /* K % g, g % S, S % 8, sizes out of range      */
    AAAC_ERR_ALIGN = 3,       /* pointer or leading dimension not aligned     */
    AAAC_ERR_UNSUPPORTED = 4, /* format / group size this build does not do  */
    AAAC_ERR_CUDA = 5,        /* a CUDA runtime error (see aaac_last_error)    */
    AAAC_ERR_WORKSPACE = 6,   /* ws is NULL or smaller than required           */
    AAAC_ERR_TIMEOUT = 7,     /* reserved: a bounded device wait ran out       */
    AAAC_ERR_COLLECTIVE = 8   /* a sharded call's reduction callback failed    */
} aaac_status;

/* Section 1 / 4: the two 4-bit layouts evaluated on the page.
 *   AAAC_INT4     : g = 128 (any power of two in [16, 256] accepted),
 *                   codebooks of 16 entries, scale stored as bf16.
 *   AAAC_NVFP4    : g = 16, codebooks of 15 entries, scale stored as FP8 E4M3
 *                   (s = e4m3_RN_satfinite(group absmax)).
 *   AAAC_NVFP4_GS : NVFP4 with a per-tensor fp32 scale, the page leaving open
 *                   whether one is used: gs = fp32_RN(max|w| / 448) in
 *                   *cfg->global_scale, the stored E4M3 factor
 *                   s8 = e4m3_RN_satfinite(fp32_RN(absmax / gs)), and the
 *                   group's scale fp32_RN(gs * s8).  Refine weights and the
 *                   round objective use s8 (gs^2 is common to every group and
 *                   multiplies err_hist once). */
typedef enum { AAAC_INT4 = 0, AAAC_NVFP4 = 1, AAAC_NVFP4_GS = 2 } aaac_format;

/* flags of aaac_config */
#define AAAC_FREEZE_T0 1u         /* never refine T0                            */
#define AAAC_FREEZE_T1 2u         /* never refine T1                            */
#define AAAC_SINGLE_CODEBOOK 4u   /* every group takes T0                       */
/* The fit and pack passes of this layer share the GPU with other layers' on
 * concurrent streams: their grids take one block per 196608 weights (at
 * least 16, never more than fill the GPU) instead of always filling it, so
 * a small layer's latency-bound rounds hold few of the SMs' block slots.
 * Results are identical with and without it. */
#define AAAC_CONCURRENT 8u

typedef struct {
    int32_t fmt;     /* aaac_format                                            */
    int32_t g;       /* scale group size along K                               */
    int32_t S;       /* selection group size: S % 8 == 0, g % S == 0           */
    int32_t iters;   /* assign+refine rounds of aaac_fit_layer, >= 0           */
    uint32_t flags;  /* AAAC_FREEZE_T0 | AAAC_FREEZE_T1 | AAAC_SINGLE_CODEBOOK
                      * | AAAC_CONCURRENT                                      */
    float* global_scale; /* AAAC_NVFP4_GS only (else ignored): device fp32 [1],
                          * 4-byte aligned; aaac_init_codebooks writes gs there,
                          * every other call reads it */
} aaac_config;

/* flags of aaac_importance */
#define AAAC_IMPORTANCE_ACCUMULATE 1u /* I_out = fp32_RN(I_in + sum), I_in read from I */
#define AAAC_IMPORTANCE_EXACT 2u      /* take the exact path for every column          */

/* Device-side statistics written by aaac_fit_layer (one struct, device memory). */
typedef struct {
    int64_t near_ties;      /* groups with |D1-D0| < 1e-6 max(D0,D1), last round  */
    int64_t groups_t1;      /* selection groups on T1, last round                 */
    int64_t empty_cells;    /* unfrozen entries left unchanged at the last refine */
    int64_t dead_groups;    /* scale groups with s == 0 or non-finite 1/s         */
    int64_t exact_groups;   /* groups whose choice took the exact fp64 path, all rounds */
    int32_t L;              /* fixed-point exponent of the centroid sums          */
    int32_t reserved;
} aaac_stats;

/* Bytes of workspace that a call with this configuration needs.  T is the
 * token count of aaac_importance (0 when only the weight-side calls are used);
 * N, K describe the layer (0 when only aaac_importance is used).  One
 * workspace of the returned size serves every call on these sizes. */
size_t aaac_workspace_size(const aaac_config* cfg, int64_t N, int64_t K, int64_t T);

/* Column importance, section 2 core mechanism 2:  I_k = sum_t X[t,k]^2.
 *   X      device bf16 [T][ldx]; only the first K columns are read.
 *   I      device fp32 [K]; written, and read first when ACCUMULATE is set.
 *   flags  AAAC_IMPORTANCE_ACCUMULATE, AAAC_IMPORTANCE_EXACT.
 * The result is the exact sum rounded once to fp32 (nearest, ties to even):
 * an fp64 pass with a rigorous error bound decides every column whose bound
 * does not straddle an fp32 rounding boundary; the rest are summed exactly.
 * Requires 0 < T, 0 < K, K % 8 == 0, ldx % 8 == 0, ldx >= K. */
aaac_status aaac_importance(const void* X, int64_t T, int64_t K, int64_t ldx, uint32_t flags,
                            float* I, void* ws, size_t ws_bytes, void* stream);

/* Scales and quantile initialisation, section 2 core mechanism 4
 * (initialisation: evenly spaced quantiles of the normalised weights, T1
 * shifted by half a step), with the scale of section 1 / 4 read as
 *   INT4 : s = bf16_RN(fp32_RN(max|w| / 7))      NVFP4 : s = e4m3_RN_sat(max|w|)
 *   NVFP4_GS : gs = fp32_RN(max over W of |w| / 448) written to
 *              *cfg->global_scale, stored s8 = e4m3_RN_sat(fp32_RN(max|w| / gs)),
 *              s = fp32_RN(gs * s8)
 *   u = fp32_RN(w * fp32_RN(1/s)); groups with s == 0 or 1/s = inf have u = 0.
 *   T0[j] = u_(floor((2j+1)M / 2n)),  T1[j] = u_(min(M-1, floor((j+1)M/n)))
 * over the ascending IEEE total order of all M = N*K values, n = 16 (INT4) or
 * 15 (NVFP4).
 *   W       device bf16 [N][K]
 *   scales  device, written: bf16 [N][K/g] (INT4) or uint8 E4M3 [N][K/g] (NVFP4)
 *   T       device fp32 [2][16], written; entries j >= n are 0.
 * Requires N*K < 2^31. */
aaac_status aaac_init_codebooks(const void* W, int64_t N, int64_t K, const aaac_config* cfg,
                                void* scales, float* T, void* ws, size_t ws_bytes,
                                void* stream);

/* The alternating fit, section 2 core mechanisms 2 and 4: cfg->iters rounds of
 *   assign : u's nearest entry in each codebook (exact distance, lowest index
 *            on a tie); per selection group of S weights
 *            D_c = sum I_k (u - T_c[q])^2, choice = (D_1 < D_0) decided exactly
 *            as by sequential fp64 arithmetic;
 *   refine : each unfrozen entry becomes the I*s^2-weighted centroid of its
 *            cell, T = sum A u / sum A with A = I_k s^2, both sums exact
 *            integer fixed point; an empty cell keeps its value; each
 *            codebook is then sorted ascending.
 *   W, scales  as written by aaac_init_codebooks (sign bits ignored)
 *   I          device fp32 [K]
 *   T          device fp32 [2][16]: in the start codebooks, out the fitted ones
 *   err_hist   device fp64 [iters]: sum over groups of s^2 * D_choice at the
 *              assign of each round (may be NULL)
 *   stats      device aaac_stats (may be NULL)
 * Requires N*K < 2^31. */
aaac_status aaac_fit_layer(const void* W, int64_t N, int64_t K, const float* I,
                           const void* scales, const aaac_config* cfg, float* T,
                           double* err_hist, aaac_stats* stats, void* ws, size_t ws_bytes,
                           void* stream);

/* The same fit as aaac_fit_layer, for callers that cannot allocate device
 * memory -- for example code that runs where cudaMalloc is not permitted, or
 * a plugin that has no access to its host framework's allocator and so cannot
 * provide a workspace.  The paper has no counterpart to this call; it exists
 * for integration only.
 *   Arguments and results are those of aaac_fit_layer, without ws/ws_bytes.
 *   Scratch: a 256 KiB array inside the library (every GPU that loads the
 *   library holds it until the process exits).  The fit's scratch is its
 *   control block (a few KB, the same for every layer), so every layer that
 *   passes the shape checks (N*K < 2^31, rejected with AAAC_ERR_SHAPE before
 *   anything is launched) fits; a scratch need above the array would be
 *   rejected with AAAC_ERR_WORKSPACE, also before any launch.
 *   The first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture.  The
 *   address is cached with the id of the context it was taken in and looked
 *   up again when another context is current (after cudaDeviceReset, say).
 *   All calls share the one array and it keeps the previous call's contents
 *   (the call clears what must start at zero).  Calls whose work overlaps on
 *   the GPU -- concurrent streams, or concurrent host threads -- race on it:
 *   serialise them.
 *   The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *   library routine. */
aaac_status aaac_fit_layer_fixed_scratch(const void* W, int64_t N, int64_t K, const float* I,
                                         const void* scales, const aaac_config* cfg, float* T,
                                         double* err_hist, aaac_stats* stats, void* stream);

/* Storage, section 2 core mechanism 3 and section 4: T is sorted and rounded
 * to bf16, a last assign (as in the fit) runs with the bf16 tables, then
 *   T_bf16        device uint16 [2][16] (64 bytes; entries j >= n are 0)
 *   codes         device uint8 [N][K/2]: entry index, low nibble = even k
 *   scales_tagged device, like scales: the scale with its sign bit set to the
 *                 group's choice when S == g (0 when S < g)
 *   choice_bits   device uint8 [N][ceil(K/S/8)], bit j%8 of byte j/8 = choice
 *                 of selection group j (LSB first); required when S < g,
 *                 ignored (may be NULL) when S == g
 *   err_final     device fp64 [1]: sum over weights of I_k (w - s T[c][q])^2
 *                 (may be NULL) */
aaac_status aaac_pack(const void* W, int64_t N, int64_t K, const float* I, const void* scales,
                      const aaac_config* cfg, const float* T, uint16_t* T_bf16, uint8_t* codes,
                      void* scales_tagged, uint8_t* choice_bits, double* err_final, void* ws,
                      size_t ws_bytes, void* stream);

/* Inference dequantisation (section 1: the dequantised values from the
 * table decide the weights used at inference, W4A16; section 2 core mechanism
 * 3: BF16 tables, choice in the scale's sign bit or in a bitmask).  The packed
 * layer of aaac_pack back to bf16 weights:
 *   W_hat[n][k] = bf16_RN(s[n][k/g] * T_bf16[c][code[n][k]])
 * where s is the magnitude of the stored scale and c is its sign bit (S == g)
 * or bit (k/S)%8 of choice_bits[n][(k/S)/8] (S < g).  The product has at most
 * 16 significant bits, so it is exact in fp32 and rounded once.  For
 * AAAC_NVFP4_GS, s = fp32_RN(gs * s8) and
 *   W_hat[n][k] = bf16_RN(fp32_RN(s * T_bf16[c][code[n][k]])).
 *   codes, scales_tagged, choice_bits, T_bf16: as aaac_pack writes them
 *                 (choice_bits may be NULL when S == g)
 *   cfg           fmt, g and S of the packed layer (iters and flags ignored)
 *   W_hat         device uint16 (bf16 bits) [N][K]
 * No workspace.  An NVFP4 code 15 (never written by aaac_pack) reads entry 15
 * of the table, which aaac_pack sets to 0. */
aaac_status aaac_dequant(const uint8_t* codes, const void* scales_tagged,
                         const uint8_t* choice_bits, const uint16_t* T_bf16, int64_t N, int64_t K,
                         const aaac_config* cfg, uint16_t* W_hat, void* stream);

/* The W4A16 linear layer on the packed format (section 1, W4A16 inference):
 *   Y[m][n] = sum_k X[m][k] * W_hat[n][k]      (W_hat as in aaac_dequant)
 *   X   device bf16 [M][ldx] (M tokens; ldx >= K, a multiple of 8)
 *   Y   device fp32 [M][N]
 * The dequantised weights never reach memory: each kernel expands its codes
 * on the fly (a GEMV on CUDA cores up to 4 tokens; tcgen05 kernels above:
 * 5 to 32 tokens on clusters of 2 to 8 CTAs splitting K when K is a
 * multiple of 32, else a fused kernel; aaac_linear_launch_plan reports which).
 * Accumulation is fp32 in the library's order, the same on every run; every
 * result is within K * 2^-24 * sum_k |X[m][k] W_hat[n][k]| of the exact sum.
 * M in [1, 2^20].  No workspace. */
aaac_status aaac_linear(const void* X, int64_t M, int64_t ldx, const uint8_t* codes,
                        const void* scales_tagged, const uint8_t* choice_bits,
                        const uint16_t* T_bf16, int64_t N, int64_t K, const aaac_config* cfg,
                        float* Y, void* stream);

/* AWQ-style pre-scaling before the fit (section 4: AAAC combined with AWQ,
 * which scales the weights before quantisation).  For alpha = alpha16 / 16:
 *   v_k  = I_k / tokens;  p_k = v_k^(alpha16/32), the product in ascending i
 *          of v^(2^(i-5)) over the set bits i of alpha16, each power by
 *          repeated fp64 square roots;
 *   z    = sqrt(max p * min p) over channels with I_k > 0;
 *   c_k  = fp32_RN(p_k / z)  (1 where I_k is not > 0);
 *   I'_k = fp32_RN(I_k / (c_k * c_k))  (fp64);
 *   W'   = bf16_RN(fp32_RN(w * c_k)).
 * The rescaled layer (W', activations x / c) computes the same map as the
 * original up to the bf16 rounding of W', and I' is its importance vector.
 *   W         device bf16 [N][K], K a multiple of 8, N*K < 2^31
 *   I         device fp32 [K] (aaac_importance over `tokens` rows of X)
 *   tokens    > 0
 *   alpha16   in [0, 16]; 0 gives c = 1, I' = I, W' = W
 *   c, I_scaled  device fp32 [K];  W_scaled  device bf16 [N][K]
 * All pointers 16-byte aligned; outputs must not overlap the inputs.
 * Two kernels, no workspace. */
aaac_status aaac_awq_prescale(const void* W, int64_t N, int64_t K, const float* I,
                              int64_t tokens, int alpha16, float* c, float* I_scaled,
                              void* W_scaled, void* stream);

/* Bytes of workspace aaac_awq_fit needs for this config and shape (0 when
 * the config or shape is invalid): the rescaled layer (2 B per weight), one
 * candidate's packed output, and the fit's own workspace. */
size_t aaac_awq_workspace_size(const aaac_config* cfg, int64_t N, int64_t K);

/* Grid search over the pre-scaling exponent.  For each i < n_alpha, in
 * order: aaac_awq_prescale with alpha16[i], then aaac_init_codebooks,
 * aaac_fit_layer (cfg->iters rounds) and aaac_pack on the rescaled layer
 * (W', I'); err_alpha[i] receives that candidate's err_final (the
 * activation-weighted error of the rescaled layer, which equals the error
 * of W_hat'/c against W'/c in the original input space).  The first
 * candidate with the lowest err_final is kept (strict improvement over all
 * earlier ones): its c, T_bf16, codes, scales_tagged and choice_bits go to
 * the outputs, its err_final to *err_final and its position i to *best
 * (AAAC_NVFP4_GS: its tensor scale to *cfg->global_scale).
 * Everything runs on `stream` with no host synchronisation.
 *   alpha16     HOST int32 [n_alpha], each in [0, 16]; n_alpha in [1, 17]
 *   c           device fp32 [K] (deploy with activations x / c)
 *   T_bf16, codes, scales_tagged, choice_bits: as aaac_pack
 *   err_final   device fp64 [1] (may be NULL); err_alpha device fp64 [n_alpha]
 *   best        device int32 [1] (may be NULL)
 *   ws          aaac_awq_workspace_size(cfg, N, K) bytes
 * A CUDA error part way leaves the outputs of earlier candidates in place. */
aaac_status aaac_awq_fit(const void* W, int64_t N, int64_t K, const float* I, int64_t tokens,
                         const aaac_config* cfg, const int32_t* alpha16, int n_alpha, float* c,
                         uint16_t* T_bf16, uint8_t* codes, void* scales_tagged,
                         uint8_t* choice_bits, double* err_final, double* err_alpha,
                         int32_t* best, void* ws, size_t ws_bytes, void* stream);

/* Row-sharded calls: one layer's rows split over several processes (one per
 * GPU), each holding N of the layer's N_total rows (its W, scales, codes
 * rows; I is the whole K columns).  Where the unsharded call reduces over all
 * rows -- the quantile histograms, the maxima that fix the fixed-point
 * exponents, each round's refine sums and objective -- the sharded call
 * hands a buffer in its workspace to the caller's reduction, which must
 * combine it over all shards in place (an all-reduce, e.g. NCCL over
 * NVLink), enqueued on `stream`.  Every reduced quantity is an integer, so
 * the result does not depend on the reduction's order: every shard ends
 * with the tables of the unsharded call on the whole layer, bit for bit,
 * and packs its own rows exactly as the unsharded pack would.  Per fit round
 * the exchange is 69 int64 values (552 bytes).
 *   op AAAC_REDUCE_SUM_I64 / MAX_I64: int64 elements; SUM_I32 / MAX_I32: int32.
 *   The callback returns 0 on success; any other value stops the call, which
 *   returns AAAC_ERR_COLLECTIVE (work already enqueued stays enqueued).
 * Every shard must make the same calls with the same cfg, K and N_total. */
#define AAAC_REDUCE_SUM_I64 0
#define AAAC_REDUCE_MAX_I64 1
#define AAAC_REDUCE_SUM_I32 2
#define AAAC_REDUCE_MAX_I32 3
typedef int (*aaac_reduce_fn)(void* user, void* buf, int64_t count, int op, void* stream);

aaac_status aaac_init_codebooks_sharded(const void* W, int64_t N, int64_t K, int64_t N_total,
                                        const aaac_config* cfg, void* scales, float* T,
                                        aaac_reduce_fn reduce, void* user, void* ws,
                                        size_t ws_bytes, void* stream);
aaac_status aaac_fit_layer_sharded(const void* W, int64_t N, int64_t K, int64_t N_total,
                                   const float* I, const void* scales, const aaac_config* cfg,
                                   float* T, double* err_hist, aaac_stats* stats,
                                   aaac_reduce_fn reduce, void* user, void* ws, size_t ws_bytes,
                                   void* stream);
aaac_status aaac_pack_sharded(const void* W, int64_t N, int64_t K, int64_t N_total,
                              const float* I, const void* scales, const aaac_config* cfg,
                              const float* T, uint16_t* T_bf16, uint8_t* codes,
                              void* scales_tagged, uint8_t* choice_bits, double* err_final,
                              aaac_reduce_fn reduce, void* user, void* ws, size_t ws_bytes,
                              void* stream);

/* aaac_linear with a workspace.  From a token count the library chooses
 * (aaac_linear_workspace_size returns 0 below it), the layer is dequantised
 * once into the workspace (as aaac_dequant) and Y = X W_hat^T runs as a bf16
 * tcgen05 GEMM with both operands fed by TMA; the fused kernels instead
 * expand W again for every token tile.  Same contract and accuracy bound as
 * aaac_linear; with a NULL or too small workspace it is aaac_linear.
 *   ws   device, aaac_linear_workspace_size(cfg, M, N, K) bytes (N*K bf16) */
size_t aaac_linear_workspace_size(const aaac_config* cfg, int64_t M, int64_t N, int64_t K);
aaac_status aaac_linear_ws(const void* X, int64_t M, int64_t ldx, const uint8_t* codes,
                           const void* scales_tagged, const uint8_t* choice_bits,
                           const uint16_t* T_bf16, int64_t N, int64_t K, const aaac_config* cfg,
                           float* Y, void* ws, size_t ws_bytes, void* stream);

/* Device-side wait status of the current device: *flag = 1 when a bounded
 * wait inside one of the library's kernels (the tensor-core aaac_linear path)
 * has run out since the library was loaded, else 0.  A kernel whose wait ran
 * out writes NaN to its output tile and still releases its tensor memory.
 * Synchronises with the device (reads a device variable). */
aaac_status aaac_device_timeouts(uint32_t* flag);

/* Debug builds: 1 when the library was compiled with AAAC_CHECKS
 * (build.py --checks), else 0.  In such a build the fit and init kernels test
 * the indices they compute (rows, strips, work-item FIFO depth, table cells,
 * refine-bin offsets, radix slots) and record the first failure; *flag gets
 * that record (the check's code in the low byte, the offending value above
 * it), 0 when every check has held -- and always 0 in a normal build.
 * aaac_device_checks synchronises with the device (reads a device variable). */
int aaac_checked_build(void);
aaac_status aaac_device_checks(uint32_t* flag);

/* Test hook: arms one host-side fault (kind "alloc", "launch" or "sync"; NULL
 * or "" disarms).  The next call that would launch work -- on any thread --
 * returns AAAC_ERR_WORKSPACE ("alloc") or AAAC_ERR_CUDA ("launch", "sync")
 * after its argument checks, launches nothing, touches no output, and
 * disarms the fault.  The environment variable AAAC_FAULT with the same
 * kinds arms one fault when the library first runs a call.  For testing a
 * caller's error paths; nothing reaches the GPU.
 * Errors: AAAC_ERR_INVALID_ARG for an unknown kind. */
aaac_status aaac_inject_fault(const char* kind);

/* Message describing the last failed call on the calling thread ("" after a
 * successful call).  Valid until the next call on the thread. */
const char* aaac_last_error(void);

/* Library version string. */
const char* aaac_version(void);

/* Launch plan of the fit and pack passes (aaac_fit_layer, aaac_pack and their
 * row-sharded forms) for N rows x K columns of a layer of N_total rows (N_total
 * = N when it is not sharded), as those calls compute it from cfg.  A host-only
 * query: no GPU work, no device memory.  out (host int32[5]):
 *   out[0]  blocks of the pass (3 warps each)
 *   out[1]  strips of 512 columns
 *   out[2]  work items per strip (runs of out[3] rows)
 *   out[3]  rows per work item
 *   out[4]  work items one warp may take: the bound that keeps its lanes'
 *           fixed-point refine partials exact
 * Errors as the calls': AAAC_ERR_INVALID_ARG (NULL cfg or out, bad flags or
 * iters), AAAC_ERR_UNSUPPORTED / AAAC_ERR_SHAPE (format, g, S, sizes,
 * N_total < N). */
aaac_status aaac_fit_launch_plan(const aaac_config* cfg, int64_t N, int64_t K, int64_t N_total,
                                 int32_t* out);

/* The kernel aaac_linear runs for M tokens of a layer of N x K weights, and
 * the plan of the cluster kernel it uses for 5 to 32 tokens.  A host-only
 * query: no GPU work, no device memory.  out (host int32[8]):
 *   out[0]  0 GEMV (up to 4 tokens), 1 cluster kernel (5 to 32 tokens, K a
 *           multiple of 32, its shared memory within the limit), 2 the
 *           fused tcgen05 kernel (aaac_linear_ws may dequantise instead)
 *   out[1]  CTAs of a cluster; each takes a contiguous share of the K blocks
 *   out[2]  64-column K blocks of the layer
 *   out[3]  bytes per weight row staged for its scales, out[4] for its
 *           choice bits (0 when S == g)
 *   out[5]  shared memory of the 16-token kernel, out[6] of the 32-token one
 *   out[7]  the shared-memory limit the plan must keep
 * out[1..7] describe the cluster kernel whatever out[0] is.  Errors:
 * AAAC_ERR_INVALID_ARG (NULL cfg or out), AAAC_ERR_UNSUPPORTED / SHAPE as
 * aaac_linear's. */
aaac_status aaac_linear_launch_plan(const aaac_config* cfg, int64_t M, int64_t N, int64_t K,
                                    int32_t* out);

/* Number of CUDA kernels this library has launched in the process so far
 * (all threads, all devices).  A measurement aid: the difference across a
 * region counts the library's kernel launches in it. */
uint64_t aaac_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* AAAC_H */
