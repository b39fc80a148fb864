"""Thin Python binding of libaaac.so (include/aaac.h).

Argument marshalling only: torch supplies device memory and the current
stream, every step of the fit runs in the library's CUDA kernels.  There is no
CPU fallback: without the built library or a CUDA device every call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

INT4 = 0
NVFP4 = 1
NVFP4_GS = 2  # NVFP4 with a per-tensor fp32 scale
FREEZE_T0 = 1
FREEZE_T1 = 2
SINGLE_CODEBOOK = 4
CONCURRENT = 8  # grids sized by the layer's weights, for layers fitted side by side
IMPORTANCE_ACCUMULATE = 1
IMPORTANCE_EXACT = 2

STATUS = {0: "AAAC_OK", 1: "AAAC_ERR_INVALID_ARG", 2: "AAAC_ERR_SHAPE", 3: "AAAC_ERR_ALIGN",
          4: "AAAC_ERR_UNSUPPORTED", 5: "AAAC_ERR_CUDA", 6: "AAAC_ERR_WORKSPACE",
          7: "AAAC_ERR_TIMEOUT", 8: "AAAC_ERR_COLLECTIVE"}

# AAAC_CHECKED=1 selects the debugging build with device-side index checks
# (built by `python -m activation_aware_codebook_b200.csrc.build --checks`).
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libaaac_checked.so" if os.environ.get("AAAC_CHECKED") == "1"
                        else "libaaac.so")

EXPORTS = ("aaac_workspace_size", "aaac_importance", "aaac_init_codebooks", "aaac_fit_layer",
           "aaac_pack", "aaac_last_error", "aaac_version", "aaac_kernel_launches",
           "aaac_fit_layer_fixed_scratch", "aaac_dequant", "aaac_linear",
           "aaac_device_timeouts", "aaac_awq_prescale", "aaac_awq_workspace_size",
           "aaac_awq_fit", "aaac_init_codebooks_sharded", "aaac_fit_layer_sharded",
           "aaac_pack_sharded", "aaac_linear_workspace_size", "aaac_linear_ws",
           "aaac_fit_launch_plan", "aaac_linear_launch_plan", "aaac_inject_fault",
           "aaac_device_checks",
           "aaac_checked_build")


# reduction callback of the row-sharded calls: (user, buf, count, op, stream) -> 0 | error
REDUCE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                             ctypes.c_int, ctypes.c_void_p)
REDUCE_SUM_I64, REDUCE_MAX_I64, REDUCE_SUM_I32, REDUCE_MAX_I32 = 0, 1, 2, 3


class AaacError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class CConfig(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("g", ctypes.c_int32), ("S", ctypes.c_int32),
                ("iters", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("global_scale", ctypes.c_void_p)]


class CStats(ctypes.Structure):
    _fields_ = [("near_ties", ctypes.c_int64), ("groups_t1", ctypes.c_int64),
                ("empty_cells", ctypes.c_int64), ("dead_groups", ctypes.c_int64),
                ("exact_groups", ctypes.c_int64), ("L", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


STATS_BYTES = ctypes.sizeof(CStats)


@dataclasses.dataclass
class Config:
    fmt: int = INT4
    g: int = 128
    S: int = 128
    iters: int = 20
    flags: int = 0
    # NVFP4_GS: device fp32 [1] holding the per-tensor scale (init_codebooks
    # allocates it on the weights' device when it is None)
    global_scale: Optional[torch.Tensor] = None

    def c(self) -> CConfig:
        gs = self.global_scale.data_ptr() if self.global_scale is not None else None
        return CConfig(self.fmt, self.g, self.S, self.iters, self.flags, gs)

    def ensure_global_scale(self, device) -> None:
        if self.fmt == NVFP4_GS and self.global_scale is None:
            self.global_scale = torch.zeros(1, dtype=torch.float32, device=device)

    @property
    def n(self) -> int:
        return 16 if self.fmt == INT4 else 15


_lib = None


def load(path: str = LIB_PATH):
    """Load libaaac.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libaaac.so not built ({path}); run "
                           "python -m activation_aware_codebook_b200.csrc.build")
    L = ctypes.CDLL(path)
    P, i64, sz, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint32
    L.aaac_workspace_size.restype = sz
    L.aaac_workspace_size.argtypes = [P, i64, i64, i64]
    L.aaac_importance.restype = ctypes.c_int
    L.aaac_importance.argtypes = [P, i64, i64, i64, u32, P, P, sz, P]
    L.aaac_init_codebooks.restype = ctypes.c_int
    L.aaac_init_codebooks.argtypes = [P, i64, i64, P, P, P, P, sz, P]
    L.aaac_fit_layer.restype = ctypes.c_int
    L.aaac_fit_layer.argtypes = [P, i64, i64, P, P, P, P, P, P, P, sz, P]
    L.aaac_pack.restype = ctypes.c_int
    L.aaac_pack.argtypes = [P, i64, i64, P, P, P, P, P, P, P, P, P, P, sz, P]
    L.aaac_last_error.restype = ctypes.c_char_p
    L.aaac_last_error.argtypes = []
    L.aaac_version.restype = ctypes.c_char_p
    L.aaac_version.argtypes = []
    L.aaac_fit_layer_fixed_scratch.restype = ctypes.c_int
    L.aaac_fit_layer_fixed_scratch.argtypes = [P, i64, i64, P, P, P, P, P, P, P]
    L.aaac_dequant.restype = ctypes.c_int
    L.aaac_dequant.argtypes = [P, P, P, P, i64, i64, P, P, P]
    L.aaac_linear.restype = ctypes.c_int
    L.aaac_linear.argtypes = [P, i64, i64, P, P, P, P, i64, i64, P, P, P]
    L.aaac_device_timeouts.restype = ctypes.c_int
    L.aaac_device_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    L.aaac_kernel_launches.restype = ctypes.c_uint64
    L.aaac_kernel_launches.argtypes = []
    L.aaac_inject_fault.restype = ctypes.c_int
    L.aaac_inject_fault.argtypes = [ctypes.c_char_p]
    L.aaac_device_checks.restype = ctypes.c_int
    L.aaac_device_checks.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    L.aaac_checked_build.restype = ctypes.c_int
    L.aaac_checked_build.argtypes = []
    L.aaac_fit_launch_plan.restype = ctypes.c_int
    L.aaac_fit_launch_plan.argtypes = [P, i64, i64, i64, ctypes.POINTER(ctypes.c_int32)]
    L.aaac_linear_launch_plan.restype = ctypes.c_int
    L.aaac_linear_launch_plan.argtypes = [P, i64, i64, i64, ctypes.POINTER(ctypes.c_int32)]
    L.aaac_awq_prescale.restype = ctypes.c_int
    L.aaac_awq_prescale.argtypes = [P, i64, i64, P, i64, ctypes.c_int, P, P, P, P]
    L.aaac_awq_workspace_size.restype = sz
    L.aaac_awq_workspace_size.argtypes = [P, i64, i64]
    L.aaac_awq_fit.restype = ctypes.c_int
    L.aaac_awq_fit.argtypes = [P, i64, i64, P, i64, P, P, ctypes.c_int, P, P, P, P, P, P, P, P,
                               P, sz, P]
    L.aaac_linear_workspace_size.restype = sz
    L.aaac_linear_workspace_size.argtypes = [P, i64, i64, i64]
    L.aaac_linear_ws.restype = ctypes.c_int
    L.aaac_linear_ws.argtypes = [P, i64, i64, P, P, P, P, i64, i64, P, P, P, sz, P]
    R = REDUCE_FN
    L.aaac_init_codebooks_sharded.restype = ctypes.c_int
    L.aaac_init_codebooks_sharded.argtypes = [P, i64, i64, i64, P, P, P, R, P, P, sz, P]
    L.aaac_fit_layer_sharded.restype = ctypes.c_int
    L.aaac_fit_layer_sharded.argtypes = [P, i64, i64, i64, P, P, P, P, P, P, R, P, P, sz, P]
    L.aaac_pack_sharded.restype = ctypes.c_int
    L.aaac_pack_sharded.argtypes = [P, i64, i64, i64, P, P, P, P, P, P, P, P, P, R, P, P, sz, P]
    _lib = L
    return L


def device_checks() -> int:
    """The first failed device-side check of a checked build (0: none)."""
    v = ctypes.c_uint32(0)
    _check(load().aaac_device_checks(ctypes.byref(v)))
    return int(v.value)


def inject_fault(kind: Optional[str]) -> None:
    """Test hook: the next call that would launch work fails on the host
    ("alloc", "launch" or "sync"; None disarms); see aaac_inject_fault."""
    _check(load().aaac_inject_fault(None if kind is None else kind.encode()))


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(load().aaac_kernel_launches())


def _check(status: int):
    if status != 0:
        raise AaacError(status, load().aaac_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libaaac takes device tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda():
    if not torch.cuda.is_available():
        raise RuntimeError("libaaac needs a CUDA device; there is no CPU path")


def workspace_size(cfg: Optional[Config], N: int = 0, K: int = 0, T: int = 0) -> int:
    c = cfg.c() if cfg is not None else None
    return int(load().aaac_workspace_size(ctypes.byref(c) if c is not None else None, N, K, T))


LINEAR_PATHS = {0: "gemv", 1: "cluster", 2: "fused"}


def linear_launch_plan(cfg: Config, M: int, N: int, K: int) -> dict:
    """Host-only: the kernel aaac_linear runs and the cluster kernel's plan."""
    out = (ctypes.c_int32 * 8)()
    _check(load().aaac_linear_launch_plan(ctypes.byref(cfg.c()), M, N, K, out))
    keys = ("path", "cluster", "kblocks", "scale_stride", "choice_stride", "smem16", "smem32",
            "smem_limit")
    d = dict(zip(keys, list(out)))
    d["path"] = LINEAR_PATHS[d["path"]]
    return d


def fit_launch_plan(cfg: Config, N: int, K: int, N_total: Optional[int] = None) -> dict:
    """The fit/pack passes' launch plan for these sizes (host-only query)."""
    out = (ctypes.c_int32 * 5)()
    _check(load().aaac_fit_launch_plan(ctypes.byref(cfg.c()), N, K,
                                       N if N_total is None else N_total, out))
    return dict(blocks=out[0], strips=out[1], items_per_strip=out[2], item_rows=out[3],
                max_items=out[4])


def workspace(cfg: Optional[Config], N: int = 0, K: int = 0, T: int = 0,
              device="cuda") -> torch.Tensor:
    return torch.empty(workspace_size(cfg, N, K, T), dtype=torch.uint8, device=device)


def _bits16(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype in (torch.bfloat16, torch.int16, torch.uint16), t.dtype
    return t.contiguous()


def importance(X: torch.Tensor, I: Optional[torch.Tensor] = None, accumulate: bool = False,
               exact: bool = False, ws: Optional[torch.Tensor] = None, stream=None,
               ncols: Optional[int] = None) -> torch.Tensor:
    """I_k = sum_t X[t,k]^2 (fp32, exact sum rounded once).  X: [T, ldx] bf16."""
    _need_cuda()
    T, ldx = X.shape
    K = ldx if ncols is None else ncols
    if X.stride(1) != 1:
        raise ValueError("X must be row-major")
    ldx = X.stride(0)
    if I is None:
        I = torch.zeros(K, dtype=torch.float32, device=X.device)
    if ws is None:
        ws = workspace(None, 0, K, T, X.device)
    flags = (IMPORTANCE_ACCUMULATE if accumulate else 0) | (IMPORTANCE_EXACT if exact else 0)
    _check(load().aaac_importance(_ptr(X), T, K, ldx, flags, _ptr(I), _ptr(ws), ws.numel(),
                                  _stream(stream)))
    return I


def init_codebooks(W: torch.Tensor, cfg: Config, ws: Optional[torch.Tensor] = None,
                   scales: Optional[torch.Tensor] = None, T: Optional[torch.Tensor] = None,
                   stream=None):
    """Absmax scales and quantile codebooks.  Returns (scales, T[2,16])."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    sdt = torch.int16 if cfg.fmt == INT4 else torch.uint8
    if scales is None:
        scales = torch.empty(N, K // cfg.g, dtype=sdt, device=W.device)
    if T is None:
        T = torch.empty(2, 16, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = workspace(cfg, N, K, 0, W.device)
    cfg.ensure_global_scale(W.device)
    c = cfg.c()
    _check(load().aaac_init_codebooks(_ptr(W), N, K, ctypes.byref(c), _ptr(scales), _ptr(T),
                                      _ptr(ws), ws.numel(), _stream(stream)))
    return scales, T


def fit_layer(W: torch.Tensor, I: torch.Tensor, scales: torch.Tensor, T: torch.Tensor,
              cfg: Config, ws: Optional[torch.Tensor] = None,
              err_hist: Optional[torch.Tensor] = None, stats: Optional[torch.Tensor] = None,
              stream=None):
    """cfg.iters assign/refine rounds; T [2,16] fp32 is updated in place.
    Returns (T, err_hist[iters] fp64, stats bytes)."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    if err_hist is None:
        err_hist = torch.zeros(max(cfg.iters, 1), dtype=torch.float64, device=W.device)
    if stats is None:
        stats = torch.zeros(STATS_BYTES, dtype=torch.uint8, device=W.device)
    if ws is None:
        ws = workspace(cfg, N, K, 0, W.device)
    c = cfg.c()
    _check(load().aaac_fit_layer(_ptr(W), N, K, _ptr(I), _ptr(scales), ctypes.byref(c), _ptr(T),
                                 _ptr(err_hist), _ptr(stats), _ptr(ws), ws.numel(),
                                 _stream(stream)))
    return T, err_hist, stats


def fit_layer_fixed_scratch(W: torch.Tensor, I: torch.Tensor, scales: torch.Tensor,
                            T: torch.Tensor, cfg: Config, err_hist: Optional[torch.Tensor] = None,
                            stats: Optional[torch.Tensor] = None, stream=None):
    """fit_layer for callers that cannot allocate: the library's own fixed
    scratch replaces the workspace (see aaac_fit_layer_fixed_scratch)."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    if err_hist is None:
        err_hist = torch.zeros(max(cfg.iters, 1), dtype=torch.float64, device=W.device)
    if stats is None:
        stats = torch.zeros(STATS_BYTES, dtype=torch.uint8, device=W.device)
    c = cfg.c()
    _check(load().aaac_fit_layer_fixed_scratch(_ptr(W), N, K, _ptr(I), _ptr(scales),
                                               ctypes.byref(c), _ptr(T), _ptr(err_hist),
                                               _ptr(stats), _stream(stream)))
    return T, err_hist, stats


def decode_stats(stats: torch.Tensor) -> dict:
    raw = bytes(stats.cpu().numpy().tobytes())
    s = CStats.from_buffer_copy(raw)
    return {f: getattr(s, f) for f, _ in CStats._fields_ if f != "reserved"}


def pack(W: torch.Tensor, I: torch.Tensor, scales: torch.Tensor, T: torch.Tensor, cfg: Config,
         ws: Optional[torch.Tensor] = None, out: Optional[dict] = None, stream=None) -> dict:
    """bf16 tables, final assign, 4-bit codes, sign-tagged scales, choice bits."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    dev = W.device
    if out is None:
        nb = (K // cfg.S + 7) // 8
        out = dict(T_bf16=torch.zeros(2, 16, dtype=torch.int16, device=dev),
                   codes=torch.empty(N, K // 2, dtype=torch.uint8, device=dev),
                   scales_tagged=torch.empty_like(scales),
                   choice_bits=(torch.empty(N, nb, dtype=torch.uint8, device=dev)
                                if cfg.S != cfg.g else None),
                   err_final=torch.zeros(1, dtype=torch.float64, device=dev))
    if ws is None:
        ws = workspace(cfg, N, K, 0, dev)
    c = cfg.c()
    _check(load().aaac_pack(_ptr(W), N, K, _ptr(I), _ptr(scales), ctypes.byref(c), _ptr(T),
                            _ptr(out["T_bf16"]), _ptr(out["codes"]), _ptr(out["scales_tagged"]),
                            _ptr(out["choice_bits"]), _ptr(out["err_final"]), _ptr(ws),
                            ws.numel(), _stream(stream)))
    return out


def device_timeouts() -> int:
    """1 when a bounded device wait of the library's kernels has run out since
    the library was loaded on the current device, else 0."""
    v = ctypes.c_uint32(0)
    _check(load().aaac_device_timeouts(ctypes.byref(v)))
    return int(v.value)


def dequant(packed: dict, cfg: Config, N: int, K: int, out: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """bf16 weights of a packed layer (the dict pack() returns), [N, K] bf16 bits (int16)."""
    _need_cuda()
    dev = packed["codes"].device
    if out is None:
        out = torch.empty(N, K, dtype=torch.int16, device=dev)
    c = cfg.c()
    _check(load().aaac_dequant(_ptr(packed["codes"]), _ptr(packed["scales_tagged"]),
                               _ptr(packed.get("choice_bits")), _ptr(packed["T_bf16"]), N, K,
                               ctypes.byref(c), _ptr(out), _stream(stream)))
    return out


def linear_workspace_size(cfg: Config, M: int, N: int, K: int) -> int:
    """Bytes of the workspace that lets linear() dequantise once (0 when the
    fused kernels are used for this token count)."""
    c = cfg.c()
    return int(load().aaac_linear_workspace_size(ctypes.byref(c), M, N, K))


def linear(X: torch.Tensor, packed: dict, cfg: Config, N: int, K: int,
           out: Optional[torch.Tensor] = None, stream=None,
           ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """W4A16 linear on a packed layer: Y[M, N] = X[M, K] @ W_hat^T, fp32.
    With a workspace (linear_workspace_size bytes) large token counts
    dequantise W once and use the TMA-fed tensor-core GEMM."""
    _need_cuda()
    assert X.dtype in (torch.bfloat16, torch.int16, torch.uint16), X.dtype
    if X.stride(1) != 1 or X.stride(0) % 8:
        X = X.contiguous()
    M, ldx = X.shape[0], X.stride(0)
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32, device=X.device)
    c = cfg.c()
    if ws is not None:
        _check(load().aaac_linear_ws(_ptr(X), M, ldx, _ptr(packed["codes"]),
                                     _ptr(packed["scales_tagged"]),
                                     _ptr(packed.get("choice_bits")), _ptr(packed["T_bf16"]), N,
                                     K, ctypes.byref(c), _ptr(out), _ptr(ws), ws.numel(),
                                     _stream(stream)))
        return out
    _check(load().aaac_linear(_ptr(X), M, ldx, _ptr(packed["codes"]),
                              _ptr(packed["scales_tagged"]), _ptr(packed.get("choice_bits")),
                              _ptr(packed["T_bf16"]), N, K, ctypes.byref(c), _ptr(out),
                              _stream(stream)))
    return out


def run_layer(W: torch.Tensor, X: torch.Tensor, cfg: Config, ws: Optional[torch.Tensor] = None,
              stream=None) -> dict:
    """importance -> init -> fit -> pack for one linear, all on the GPU."""
    N, K = W.shape
    if ws is None:
        ws = workspace(cfg, N, K, X.shape[0], W.device)
    I = importance(X, ws=ws, stream=stream)
    scales, T = init_codebooks(W, cfg, ws=ws, stream=stream)
    T_init = T.clone()
    T, err_hist, stats = fit_layer(W, I, scales, T, cfg, ws=ws, stream=stream)
    out = pack(W, I, scales, T, cfg, ws=ws, stream=stream)
    out.update(global_scale=cfg.global_scale)
    out.update(I=I, scales=scales, T_init=T_init, T=T, err_hist=err_hist[:cfg.iters],
               stats=stats)
    return out


def awq_prescale(W: torch.Tensor, I: torch.Tensor, tokens: int, alpha16: int, stream=None):
    """AWQ-style pre-scaling for alpha = alpha16 / 16: (c, I', W') -- the
    per-input-channel scales, the importance of the activations x / c, and
    the rescaled bf16 weights (int16 bits)."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    dev = W.device
    c = torch.empty(K, dtype=torch.float32, device=dev)
    Is = torch.empty(K, dtype=torch.float32, device=dev)
    Ws = torch.empty(N, K, dtype=torch.int16, device=dev)
    _check(load().aaac_awq_prescale(_ptr(W), N, K, _ptr(I), int(tokens), int(alpha16), _ptr(c),
                                    _ptr(Is), _ptr(Ws), _stream(stream)))
    return c, Is, Ws


def awq_fit(W: torch.Tensor, I: torch.Tensor, tokens: int, cfg: Config, alphas16,
            ws: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Grid search over alpha = j/16 for j in alphas16: pre-scale, fit and
    pack each candidate on the device and keep the first with the lowest
    err_final.  Returns the kept packed layer, c, err_final, the err_final of
    every candidate (err_alpha) and the kept position (best), on the device."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    dev = W.device
    js = (ctypes.c_int32 * len(alphas16))(*[int(j) for j in alphas16])
    cfg.ensure_global_scale(dev)
    c_cfg = cfg.c()
    if ws is None:
        need = load().aaac_awq_workspace_size(ctypes.byref(c_cfg), N, K)
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    G = K // cfg.g
    sdt = torch.int16 if cfg.fmt == INT4 else torch.uint8
    nb = (K // cfg.S + 7) // 8
    out = dict(c=torch.empty(K, dtype=torch.float32, device=dev),
               T_bf16=torch.zeros(2, 16, dtype=torch.int16, device=dev),
               codes=torch.empty(N, K // 2, dtype=torch.uint8, device=dev),
               scales_tagged=torch.empty(N, G, dtype=sdt, device=dev),
               choice_bits=(torch.empty(N, nb, dtype=torch.uint8, device=dev)
                            if cfg.S != cfg.g else None),
               err_final=torch.zeros(1, dtype=torch.float64, device=dev),
               err_alpha=torch.zeros(len(alphas16), dtype=torch.float64, device=dev),
               best=torch.full((1,), -1, dtype=torch.int32, device=dev))
    _check(load().aaac_awq_fit(_ptr(W), N, K, _ptr(I), int(tokens), ctypes.byref(c_cfg), js,
                               len(alphas16), _ptr(out["c"]), _ptr(out["T_bf16"]),
                               _ptr(out["codes"]), _ptr(out["scales_tagged"]),
                               _ptr(out["choice_bits"]), _ptr(out["err_final"]),
                               _ptr(out["err_alpha"]), _ptr(out["best"]), _ptr(ws), ws.numel(),
                               _stream(stream)))
    return out


# --------------------------------------------------------------------------
# row-sharded calls (one layer's rows over several processes / GPUs)
# --------------------------------------------------------------------------
class ShardReducer:
    """Adapts a Python all-reduce to the library's callback.  The library
    hands a buffer inside the workspace `ws`; `allreduce(t, op)` receives a
    torch view of it (int64 or int32) and op "sum" or "max", and must combine
    it in place over all shards on the current stream (for example
    torch.distributed.all_reduce with NCCL)."""

    def __init__(self, ws: torch.Tensor, allreduce):
        self.ws, self.allreduce, self.error = ws, allreduce, None

        def cb(user, buf, count, op, stream):
            try:
                off = int(buf) - self.ws.data_ptr()
                esz = 8 if op in (REDUCE_SUM_I64, REDUCE_MAX_I64) else 4
                dt = torch.int64 if esz == 8 else torch.int32
                assert 0 <= off and off + count * esz <= self.ws.numel()
                t = self.ws[off:off + count * esz].view(dt)
                self.allreduce(t, "sum" if op in (REDUCE_SUM_I64, REDUCE_SUM_I32) else "max")
                return 0
            except Exception as e:  # reported by the call as AAAC_ERR_COLLECTIVE
                self.error = e
                return 1

        self.fn = REDUCE_FN(cb)  # kept alive with the reducer

    def check(self, status: int):
        if status == 8 and self.error is not None:
            raise AaacError(status, f"reduce callback failed: {self.error!r}")
        _check(status)


def torch_allreduce(group=None):
    """An allreduce for ShardReducer over torch.distributed (NCCL on GPUs)."""
    import torch.distributed as dist

    def run(t, op):
        dist.all_reduce(t, op=dist.ReduceOp.SUM if op == "sum" else dist.ReduceOp.MAX,
                        group=group)
    return run


def init_codebooks_sharded(W: torch.Tensor, N_total: int, cfg: Config, allreduce,
                           ws: Optional[torch.Tensor] = None, stream=None):
    """init_codebooks over a layer whose rows are split over shards; this
    shard holds W [N, K].  Returns (scales [N, K/g], T [2, 16]); T is the
    whole layer's quantile initialisation on every shard."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    sdt = torch.int16 if cfg.fmt == INT4 else torch.uint8
    scales = torch.empty(N, K // cfg.g, dtype=sdt, device=W.device)
    T = torch.empty(2, 16, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = workspace(cfg, N, K, 0, W.device)
    cfg.ensure_global_scale(W.device)
    red = ShardReducer(ws, allreduce)
    c = cfg.c()
    red.check(load().aaac_init_codebooks_sharded(_ptr(W), N, K, int(N_total), ctypes.byref(c),
                                                 _ptr(scales), _ptr(T), red.fn, None, _ptr(ws),
                                                 ws.numel(), _stream(stream)))
    return scales, T


def fit_layer_sharded(W: torch.Tensor, N_total: int, I: torch.Tensor, scales: torch.Tensor,
                      T: torch.Tensor, cfg: Config, allreduce, ws: Optional[torch.Tensor] = None,
                      stream=None):
    """fit_layer over a row-sharded layer.  Returns (T, err_hist, stats); every
    shard gets the whole layer's tables, history and counters."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    err_hist = torch.zeros(max(cfg.iters, 1), dtype=torch.float64, device=W.device)
    stats = torch.zeros(STATS_BYTES, dtype=torch.uint8, device=W.device)
    if ws is None:
        ws = workspace(cfg, N, K, 0, W.device)
    red = ShardReducer(ws, allreduce)
    c = cfg.c()
    red.check(load().aaac_fit_layer_sharded(_ptr(W), N, K, int(N_total), _ptr(I), _ptr(scales),
                                            ctypes.byref(c), _ptr(T), _ptr(err_hist),
                                            _ptr(stats), red.fn, None, _ptr(ws), ws.numel(),
                                            _stream(stream)))
    return T, err_hist, stats


def pack_sharded(W: torch.Tensor, N_total: int, I: torch.Tensor, scales: torch.Tensor,
                 T: torch.Tensor, cfg: Config, allreduce, ws: Optional[torch.Tensor] = None,
                 stream=None) -> dict:
    """pack of this shard's rows; err_final is the whole layer's."""
    _need_cuda()
    W = _bits16(W)
    N, K = W.shape
    dev = W.device
    nb = (K // cfg.S + 7) // 8
    out = dict(T_bf16=torch.zeros(2, 16, dtype=torch.int16, device=dev),
               codes=torch.empty(N, K // 2, dtype=torch.uint8, device=dev),
               scales_tagged=torch.empty_like(scales),
               choice_bits=(torch.empty(N, nb, dtype=torch.uint8, device=dev)
                            if cfg.S != cfg.g else None),
               err_final=torch.zeros(1, dtype=torch.float64, device=dev))
    if ws is None:
        ws = workspace(cfg, N, K, 0, dev)
    red = ShardReducer(ws, allreduce)
    c = cfg.c()
    red.check(load().aaac_pack_sharded(_ptr(W), N, K, int(N_total), _ptr(I), _ptr(scales),
                                       ctypes.byref(c), _ptr(T), _ptr(out["T_bf16"]),
                                       _ptr(out["codes"]), _ptr(out["scales_tagged"]),
                                       _ptr(out["choice_bits"]), _ptr(out["err_final"]),
                                       red.fn, None, _ptr(ws), ws.numel(), _stream(stream)))
    return out
