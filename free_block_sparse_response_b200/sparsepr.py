"""Python binding of libsparsepr (the SparsePR C ABI in include/sparsepr.h).

Argument marshalling only: torch provides device memory and the current stream, every
step of the attention call runs in the library's CUDA kernels.  There is no CPU or
PyTorch fallback: if the library is not built, or no GPU is present, calls raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import NamedTuple, Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsparsepr.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NONFINITE = range(6)
BF16, F32 = 0, 1
WEIGHT_INV_NORM, WEIGHT_UNIFORM = 0, 1
RIDGE_RELATIVE = 0x100  # weight_mode option bit: lambda relative to tr(X_c^T W X_c) / d
PARTITION_RESPONSE, PARTITION_SEMANTIC = 0, 1
ROUTE_CENTROID, ROUTE_SIZE_CORRECTED, ROUTE_LSE = 0, 1, 2
BUDGET_UNIFORM, BUDGET_GLOBAL = 0, 1
_DTYPE_CODE = {torch.bfloat16: BF16, torch.float32: F32}

EXPORTED_SYMBOLS = (
    "sparsepr_num_groups", "sparsepr_route_k", "sparsepr_probe_rows", "sparsepr_workspace_size",
    "sparsepr_partition", "sparsepr_route", "sparsepr_sparse_attn", "sparsepr_dense_attn",
    "sparsepr_probe_dense", "sparsepr_fit_residual", "sparsepr_apply_residual", "sparsepr_check",
    "sparsepr_last_error", "sparsepr_test_fill_workspace_size", "sparsepr_test_fill",
    "sparsepr_test_topk", "sparsepr_row_errors", "sparsepr_launch_count", "sparsepr_fit_residual_noalloc",
    "sparsepr_kernel_timing", "sparsepr_kernel_timing_read",
    "sparsepr_sparse_attn_apply", "sparsepr_reset_workspace", "sparsepr_call_workspace_size", "sparsepr_attention",
    "sparsepr_host_workspace_size", "sparsepr_attention_host", "sparsepr_test_partition_trace",
)


class SparsePRError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"[sparsepr error {code}] {message}")
        self.code = code


class _CParams(ctypes.Structure):
    _fields_ = [("block", ctypes.c_int32), ("n_sampled", ctypes.c_int32), ("n_probe", ctypes.c_int32),
                ("kmeans_iters", ctypes.c_int32), ("rank", ctypes.c_int32), ("weight_mode", ctypes.c_int32),
                ("density", ctypes.c_double), ("ridge_lambda", ctypes.c_double), ("scale", ctypes.c_float),
                ("partition_mode", ctypes.c_int32), ("route_scores", ctypes.c_int32),
                ("route_budget", ctypes.c_int32)]


@dataclasses.dataclass(frozen=True)
class SparsePRConfig:
    """Parameters of one call: block B, sampled queries S, probe rows P, k-means
    iterations T, subspace rank r, probe weighting, density rho, ridge lambda, scale,
    the partition rule (PARTITION_RESPONSE, or the PARTITION_SEMANTIC baseline), the
    block-routing score (ROUTE_CENTROID, ROUTE_SIZE_CORRECTED or ROUTE_LSE) and the split
    of the pair budget (BUDGET_UNIFORM: k groups per block; BUDGET_GLOBAL: one budget
    per head, spent on the best pairs)."""
    block: int = 128
    n_sampled: int = 512
    n_probe: int = 256
    kmeans_iters: int = 4
    rank: int = 32
    weight_mode: int = WEIGHT_INV_NORM
    density: float = 0.22
    ridge_lambda: float = 1e-3
    scale: float = 0.0
    partition_mode: int = 0
    route_scores: int = 0
    route_budget: int = 0

    def c(self) -> _CParams:
        return _CParams(self.block, self.n_sampled, self.n_probe, self.kmeans_iters, self.rank,
                        self.weight_mode, self.density, self.ridge_lambda, self.scale, self.partition_mode,
                        self.route_scores, self.route_budget)


_LIB = None
_vp, _i32, _i64p, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_float


def lib() -> ctypes.CDLL:
    """Load libsparsepr.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        _LIB = load_library(LIB_PATH)
    return _LIB


def load_library(path: str) -> ctypes.CDLL:
    """Open a build of the library at ``path`` with every entry point's signature set
    (``lib()`` opens the default build; the tests also open the wait-limit build)."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m free_block_sparse_response_b200.build`")
    L = ctypes.CDLL(path)
    P = ctypes.POINTER(_CParams)
    sig = {
        "sparsepr_num_groups": (_i32, [_i32, _i32]),
        "sparsepr_route_k": (_i32, [_i32, _i32, ctypes.c_double, _i32]),
        "sparsepr_probe_rows": (ctypes.c_int, [_i32, _i32, _i32, _i32, _vp, _vp]),
        "sparsepr_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32, _i32, P]),
        "sparsepr_partition": (ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, P, _vp, _vp, _vp,
                                              _vp, _vp, _vp, _vp, _vp]),
        "sparsepr_route": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i32, _i32, P, _vp, ctypes.POINTER(_i32), _vp,
                                          _vp, _vp]),
        "sparsepr_sparse_attn": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, _i32, _vp,
                                                _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _vp]),
        "sparsepr_sparse_attn_apply": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, _i32,
                                                      _vp, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _vp, _i32,
                                                      _vp, _vp, _vp, _vp]),
        "sparsepr_dense_attn": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, _i32, _f32,
                                               _vp, _vp, _vp]),
        "sparsepr_probe_dense": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, _i32, _vp,
                                                _i32, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _vp, _vp]),
        "sparsepr_fit_residual": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, ctypes.c_double, _i32,
                                                 _i32, _vp, _vp, _vp, _vp]),
        "sparsepr_apply_residual": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                                                   ctypes.c_int, _vp]),
        "sparsepr_check": (ctypes.c_int, [_vp, _vp]),
        "sparsepr_reset_workspace": (ctypes.c_int, [_vp, _vp]),
        "sparsepr_last_error": (ctypes.c_char_p, []),
        "sparsepr_test_fill_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32]),
        "sparsepr_test_fill": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
        "sparsepr_test_topk": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
        "sparsepr_row_errors": (ctypes.c_int, [_vp, ctypes.c_int, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
        "sparsepr_launch_count": (ctypes.c_uint64, []),
        "sparsepr_kernel_timing": (ctypes.c_int, [ctypes.c_int]),
        "sparsepr_kernel_timing_read": (ctypes.c_int, [_vp, _vp]),
        "sparsepr_fit_residual_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, ctypes.c_double,
                                                         _i32, _i32, _vp, _vp, _vp, _vp]),
        "sparsepr_call_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _i32, _i32, _i32, _i32, P]),
        "sparsepr_attention": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, P, _vp, _vp,
                                              _vp]),
        "sparsepr_host_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _i32, _i32, _i32, _i32, P, _i32]),
        "sparsepr_attention_host": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, P, _vp,
                                                   _i32, _vp, _vp, _vp]),
        "sparsepr_test_partition_trace": (ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32, P, _vp,
                                                         _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


def _call(name: str, *args) -> int:
    rc = getattr(lib(), name)(*args)
    if rc != OK:
        msg = lib().sparsepr_last_error().decode(errors="replace")
        raise SparsePRError(rc, f"{name}: {msg}")
    return rc


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _need_cuda(*ts: torch.Tensor) -> None:
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("SparsePR tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("SparsePR tensors must be contiguous")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")
    return _DTYPE_CODE[t.dtype]


# ------------------------------------------------------------------------ host helpers

def num_groups(n: int, block: int) -> int:
    return int(lib().sparsepr_num_groups(n, block))


def route_k(n: int, block: int, density: float, n_probe: int) -> int:
    return int(lib().sparsepr_route_k(n, block, density, n_probe))


def workspace_size(batch: int, heads: int, n: int, d: int, cfg: SparsePRConfig) -> int:
    size = int(lib().sparsepr_workspace_size(batch, heads, n, d, ctypes.byref(cfg.c())))
    if size == 0:
        raise SparsePRError(ERR_INVALID_ARG, "invalid sizes for the workspace")
    return size


def new_workspace(batch: int, heads: int, n: int, d: int, cfg: SparsePRConfig, device) -> torch.Tensor:
    """Workspace for calls of these sizes; its 256-byte status header starts at zero."""
    ws = torch.empty(workspace_size(batch, heads, n, d, cfg), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def check(ws: torch.Tensor) -> None:
    """Wait for the current stream and raise if a device-side error was recorded."""
    _call("sparsepr_check", _p(ws), _stream(ws))


def reset_workspace(ws: torch.Tensor) -> None:
    """Clear the workspace header (status word and the record of the key-group K/V copy)."""
    _call("sparsepr_reset_workspace", _p(ws), _stream(ws))


# ----------------------------------------------------------------------------- stages

class Partition(NamedTuple):
    key_perm: torch.Tensor      # [Bt, H, G*B] int32, -1 pads
    key_gsize: torch.Tensor     # [Bt, H, G] int32
    query_perm: torch.Tensor    # [Bt, H, G*B] int32
    qblock_size: torch.Tensor   # [Bt, H, G] int32
    block_scores: torch.Tensor  # [Bt, H, G, G] fp32


def partition(q, k, cfg: SparsePRConfig, ws: torch.Tensor, sample_idx: Optional[torch.Tensor] = None) -> Partition:
    _need_cuda(q, k, ws, sample_idx)
    bt, h, n, d = q.shape
    g = num_groups(n, cfg.block)
    dev = q.device
    out = Partition(
        torch.empty(bt, h, g * cfg.block, dtype=torch.int32, device=dev),
        torch.empty(bt, h, g, dtype=torch.int32, device=dev),
        torch.empty(bt, h, g * cfg.block, dtype=torch.int32, device=dev),
        torch.empty(bt, h, g, dtype=torch.int32, device=dev),
        torch.empty(bt, h, g, g, dtype=torch.float32, device=dev))
    _call("sparsepr_partition", _p(q), _p(k), _dtype_code(q), bt, h, n, d, ctypes.byref(cfg.c()),
          _p(sample_idx), *(_p(t) for t in out), _p(ws), _stream(q))
    return out


def route(part: Partition, n: int, cfg: SparsePRConfig, ws: torch.Tensor):
    """Returns (route [Bt,H,G,k] int32, k, executed_pairs [Bt,H] int64); under the global
    budget k = G and each row ends with -1 after its groups."""
    bt, h, g, _ = part.block_scores.shape
    # row capacity: k groups per block, or G (rows padded with -1) under the global budget
    kk = g if cfg.route_budget == BUDGET_GLOBAL else route_k(n, cfg.block, cfg.density, cfg.n_probe)
    rt = torch.empty(bt, h, g, kk, dtype=torch.int32, device=ws.device)
    pairs = torch.empty(bt, h, dtype=torch.int64, device=ws.device)
    k_out = _i32(0)
    _call("sparsepr_route", _p(part.block_scores), _p(part.key_gsize), _p(part.qblock_size), bt, h, n,
          ctypes.byref(cfg.c()), _p(rt), ctypes.byref(k_out), _p(pairs), _p(ws), _stream(ws))
    assert k_out.value == kk
    return rt, kk, pairs


def sparse_attn(q, k, v, part: Partition, rt: torch.Tensor, kk: int, cfg: SparsePRConfig,
                out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need_cuda(q, k, v, rt)
    bt, h, n, d = q.shape
    s_out = torch.empty(bt, h, n, d, dtype=torch.float32, device=q.device) if out is None else out
    _call("sparsepr_sparse_attn", _p(q), _p(k), _p(v), _dtype_code(q), bt, h, n, d, cfg.block,
          _p(part.key_perm), _p(part.key_gsize), _p(part.query_perm), _p(part.qblock_size), _p(rt), kk,
          cfg.scale, _p(s_out), _p(ws), _stream(q))
    return s_out


def fused_supported(q: torch.Tensor, cfg: SparsePRConfig) -> bool:
    """Whether the fused correction (sparse_attn_apply) is built for this shape."""
    return q.dtype == torch.bfloat16 and q.shape[-1] == 128 and cfg.block == 128


def sparse_attn_apply(q, k, v, part: Partition, rt: torch.Tensor, kk: int, cfg: SparsePRConfig, m: torch.Tensor,
                      beta: torch.Tensor, probe_idx: torch.Tensor, probe_out: torch.Tensor, ws: torch.Tensor,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Block-sparse attention with O = S + S M^T + beta formed in its epilogue, probe
    rows set to probe_out; O [Bt,H,N,d] bf16 (bf16, d = 128, B = 128)."""
    _need_cuda(q, k, v, rt, m, beta, probe_idx, probe_out, ws)
    bt, h, n, d = q.shape
    o = torch.empty(bt, h, n, d, dtype=torch.bfloat16, device=q.device) if out is None else out
    p = probe_idx.shape[-1]
    _call("sparsepr_sparse_attn_apply", _p(q), _p(k), _p(v), _dtype_code(q), bt, h, n, d, cfg.block,
          _p(part.key_perm), _p(part.key_gsize), _p(part.query_perm), _p(part.qblock_size), _p(rt), kk,
          cfg.scale, _p(m), _p(beta), _p(probe_idx), p, _p(probe_out), _p(o), _p(ws), _stream(q))
    return o


def dense_attn(q, k, v, block: int = 128, scale: float = 0.0, out: Optional[torch.Tensor] = None,
               ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dense softmax attention of every row with the same kernel family (fp32 out)."""
    _need_cuda(q, k, v, ws)
    bt, h, n, d = q.shape
    o = torch.empty(bt, h, n, d, dtype=torch.float32, device=q.device) if out is None else out
    _call("sparsepr_dense_attn", _p(q), _p(k), _p(v), _dtype_code(q), bt, h, n, d, block, scale, _p(o), _p(ws),
          _stream(q))
    return o


def probe_rows(n: int, p: int, batch: int, heads: int, device) -> torch.Tensor:
    idx = torch.empty(batch, heads, p, dtype=torch.int32, device=device)
    _call("sparsepr_probe_rows", n, p, batch, heads, _p(idx), ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream))
    return idx


def probe_dense(q, k, v, probe_idx, part: Partition, rt, kk: int, cfg: SparsePRConfig, ws: torch.Tensor):
    """Returns (probe_out, probe_sparse), each [Bt,H,P,d] fp32."""
    _need_cuda(q, k, v, probe_idx, rt, ws)
    bt, h, n, d = q.shape
    p = probe_idx.shape[-1]
    po = torch.empty(bt, h, p, d, dtype=torch.float32, device=q.device)
    ps = torch.empty_like(po)
    _call("sparsepr_probe_dense", _p(q), _p(k), _p(v), _dtype_code(q), bt, h, n, d, cfg.block, _p(probe_idx), p,
          _p(part.key_perm), _p(part.key_gsize), _p(part.query_perm), _p(rt), kk, cfg.scale, _p(po), _p(ps),
          _p(ws), _stream(q))
    return po, ps


def fit_residual(probe_sparse, probe_out, cfg: SparsePRConfig, ws: torch.Tensor,
                 weights: Optional[torch.Tensor] = None):
    """Returns (M [Bt,H,d,d], beta [Bt,H,d]) fp32."""
    _need_cuda(probe_sparse, probe_out, ws, weights)
    bt, h, p, d = probe_out.shape
    m = torch.empty(bt, h, d, d, dtype=torch.float32, device=probe_out.device)
    beta = torch.empty(bt, h, d, dtype=torch.float32, device=probe_out.device)
    _call("sparsepr_fit_residual", _p(probe_sparse), _p(probe_out), _p(weights), bt, h, d, p, cfg.ridge_lambda,
          cfg.rank, cfg.weight_mode, _p(m), _p(beta), _p(ws), _stream(probe_out))
    return m, beta


def fit_residual_noalloc(probe_sparse, probe_out, cfg: SparsePRConfig, m: torch.Tensor, beta: torch.Tensor,
                         weights: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None):
    """The fit through the allocation-free entry point, for callers that cannot
    allocate device memory during the call: results go to the caller's m [Bt,H,d,d]
    and beta [Bt,H,d]; scratch is the library's fixed static array (no workspace).
    ``status``, a one-element int32 device tensor, receives the call's device status."""
    _need_cuda(probe_sparse, probe_out, m, beta, weights, status)
    bt, h, p, d = probe_out.shape
    _call("sparsepr_fit_residual_noalloc", _p(probe_sparse), _p(probe_out), _p(weights), bt, h, d, p,
          cfg.ridge_lambda, cfg.rank, cfg.weight_mode, _p(m), _p(beta), _p(status), _stream(probe_out))
    return m, beta


def apply_residual(s_out, m, beta, probe_idx, probe_out, out_dtype=torch.bfloat16,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need_cuda(s_out, m, beta, probe_idx, probe_out)
    bt, h, n, d = s_out.shape
    p = probe_idx.shape[-1]
    o = torch.empty(bt, h, n, d, dtype=out_dtype, device=s_out.device) if out is None else out
    _call("sparsepr_apply_residual", _p(s_out), _p(m), _p(beta), _p(probe_idx), _p(probe_out), bt, h, n, d, p,
          _p(o), _DTYPE_CODE[o.dtype], _stream(s_out))
    return o


# --------------------------------------------------------------------------- the call

def attention(q, k, v, cfg: SparsePRConfig, ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
              return_parts: bool = False, fused: Optional[bool] = None):
    """One SparsePR attention call.  Returns O [Bt,H,N,d] in q's dtype (and the
    intermediates if asked).  Asynchronous on the current stream; ``check(ws)`` surfaces
    device-side errors.

    fused (default: when built for the shape and no intermediates are asked for):
    partition, route, probe rows, fit, then the sparse attention with the correction in
    its epilogue (S never leaves the SM).  Otherwise: partition, route, sparse attention
    (S fp32), probe rows, fit, apply."""
    _need_cuda(q, k, v)
    bt, h, n, d = q.shape
    if ws is None:
        ws = new_workspace(bt, h, n, d, cfg, q.device)
    if fused is None:
        fused = not return_parts and fused_supported(q, cfg)
    part = partition(q, k, cfg, ws)
    rt, kk, pairs = route(part, n, cfg, ws)
    pidx = probe_rows(n, cfg.n_probe, bt, h, q.device)
    s_out = None
    if not fused:
        s_out = sparse_attn(q, k, v, part, rt, kk, cfg, ws=ws)
    p_out, p_sparse = probe_dense(q, k, v, pidx, part, rt, kk, cfg, ws)
    m, beta = fit_residual(p_sparse, p_out, cfg, ws)
    if fused:
        o = sparse_attn_apply(q, k, v, part, rt, kk, cfg, m, beta, pidx, p_out, ws, out=out)
    else:
        o = apply_residual(s_out, m, beta, pidx, p_out, out_dtype=q.dtype, out=out)
    if not return_parts:
        return o
    return o, {"partition": part, "route": rt, "k": kk, "executed_pairs": pairs, "S": s_out, "probe_idx": pidx,
               "probe_out": p_out, "probe_sparse": p_sparse, "M": m, "beta": beta, "ws": ws}


# ------------------------------------------------------------------------ measurement

def row_errors(o: torch.Tensor, o_ref: torch.Tensor, probe_idx: Optional[torch.Tensor]) -> torch.Tensor:
    """Per-row relative L2 error of o against o_ref ([Bt,H,N] fp32, NaN on probe rows)."""
    _need_cuda(o, o_ref, probe_idx)
    bt, h, n, d = o.shape
    p = 0 if probe_idx is None else probe_idx.shape[-1]
    err = torch.empty(bt, h, n, dtype=torch.float32, device=o.device)
    _call("sparsepr_row_errors", _p(o), _DTYPE_CODE[o.dtype], _p(o_ref), _p(probe_idx), bt, h, n, d, p, _p(err),
          _stream(o))
    return err


def kernel_timing(enable: bool) -> None:
    """Record CUDA events around every later attention kernel (measurement hook)."""
    _call("sparsepr_kernel_timing", 1 if enable else 0)


def kernel_timing_read():
    """(summed ms, launches) of the attention kernels timed since the last read."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int64(0)
    _call("sparsepr_kernel_timing_read", ctypes.byref(ms), ctypes.byref(n))
    return ms.value, n.value


def launch_count() -> int:
    """Kernels the library has enqueued since it was loaded."""
    return int(lib().sparsepr_launch_count())


# ------------------------------------------------------- decision kernels, injected input

def test_fill(dist: torch.Tensor, cap: int) -> torch.Tensor:
    """Capacity fill on injected fp32 distances [H, n, G] -> labels [H, n] int32."""
    _need_cuda(dist)
    h, n, g = dist.shape
    ws = torch.empty(int(lib().sparsepr_test_fill_workspace_size(h, n, g)), dtype=torch.uint8, device=dist.device)
    labels = torch.empty(h, n, dtype=torch.int32, device=dist.device)
    _call("sparsepr_test_fill", _p(dist), h, n, g, cap, _p(labels),
          _p(ws), _stream(dist))
    check(ws)
    return labels


def test_topk(scores: torch.Tensor, k: int) -> torch.Tensor:
    """Routing selection on injected fp32 scores [H, Gq, G] -> route [H, Gq, k] int32."""
    _need_cuda(scores)
    h, gq, g = scores.shape
    ws = torch.zeros(256, dtype=torch.uint8, device=scores.device)
    rt = torch.empty(h, gq, k, dtype=torch.int32, device=scores.device)
    _call("sparsepr_test_topk", _p(scores), h, gq, g, k, _p(rt), _p(ws), _stream(scores))
    check(ws)
    return rt


class _CTrace(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in ("sample_idx", "key_gamma", "key_dist", "key_labels", "mu",
                                                      "query_gamma", "query_dist", "query_labels", "qbar")]


def test_partition_trace(q, k, cfg: SparsePRConfig, ws: Optional[torch.Tensor] = None, dists: bool = True):
    """sparsepr_partition with its internal state captured: returns (Partition, dict of
    device tensors: sample_idx [S], key_gamma / query_gamma [Bt*H,d,d], key_dist /
    query_dist [T,Bt*H,N,G] (only when ``dists``), key_labels / query_labels [T,Bt*H,N],
    mu / qbar [Bt*H,G,d])."""
    _need_cuda(q, k, ws)
    bt, h, n, d = q.shape
    g, t, hh, dev = num_groups(n, cfg.block), cfg.kmeans_iters, bt * h, q.device
    ws = new_workspace(bt, h, n, d, cfg, dev) if ws is None else ws
    f32, i32 = torch.float32, torch.int32
    tr = {"sample_idx": torch.empty(cfg.n_sampled, dtype=i32, device=dev),
          "key_gamma": torch.empty(hh, d, d, dtype=f32, device=dev),
          "key_labels": torch.empty(t, hh, n, dtype=i32, device=dev),
          "mu": torch.empty(hh, g, d, dtype=f32, device=dev),
          "query_gamma": torch.empty(hh, d, d, dtype=f32, device=dev),
          "query_labels": torch.empty(t, hh, n, dtype=i32, device=dev),
          "qbar": torch.empty(hh, g, d, dtype=f32, device=dev)}
    if dists:
        tr["key_dist"] = torch.empty(t, hh, n, g, dtype=f32, device=dev)
        tr["query_dist"] = torch.empty(t, hh, n, g, dtype=f32, device=dev)
    ct = _CTrace(**{name: (tr[name].data_ptr() if name in tr and tr[name].numel() else None)
                    for name, _ in _CTrace._fields_})
    out = Partition(
        torch.empty(bt, h, g * cfg.block, dtype=i32, device=dev), torch.empty(bt, h, g, dtype=i32, device=dev),
        torch.empty(bt, h, g * cfg.block, dtype=i32, device=dev), torch.empty(bt, h, g, dtype=i32, device=dev),
        torch.empty(bt, h, g, g, dtype=f32, device=dev))
    _call("sparsepr_test_partition_trace", _p(q), _p(k), _dtype_code(q), bt, h, n, d, ctypes.byref(cfg.c()), None,
          *(_p(x) for x in out), ctypes.byref(ct), _p(ws), _stream(q))
    check(ws)
    return out, tr


# ------------------------------------------------------------------ one-call entry points

def call_workspace(q: torch.Tensor, cfg: SparsePRConfig) -> torch.Tensor:
    """Workspace of the one-call entry ``attention_call`` (header zeroed)."""
    bt, h, n, d = q.shape
    size = int(lib().sparsepr_call_workspace_size(_dtype_code(q), bt, h, n, d, ctypes.byref(cfg.c())))
    if size == 0:
        raise SparsePRError(ERR_INVALID_ARG, "invalid sizes or parameters for the call")
    ws = torch.empty(size, dtype=torch.uint8, device=q.device)
    ws[:256].zero_()
    return ws


def attention_call(q, k, v, cfg: SparsePRConfig, ws: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The whole call as one native entry point (``sparsepr_attention``): the same stages
    and order as ``attention``, every intermediate in ``ws``."""
    _need_cuda(q, k, v)
    bt, h, n, d = q.shape
    ws = call_workspace(q, cfg) if ws is None else ws
    o = torch.empty_like(q) if out is None else out
    _call("sparsepr_attention", _p(q), _p(k), _p(v), _dtype_code(q), bt, h, n, d, ctypes.byref(cfg.c()), _p(o),
          _p(ws), _stream(q))
    return o


_COPY_STREAMS = {}


def host_workspace(q: torch.Tensor, cfg: SparsePRConfig, groups: int, device=None) -> torch.Tensor:
    """Device workspace of ``attention_host`` for host tensors shaped like q."""
    bt, h, n, d = q.shape
    size = int(lib().sparsepr_host_workspace_size(_dtype_code(q), bt, h, n, d, ctypes.byref(cfg.c()), groups))
    if size == 0:
        raise SparsePRError(ERR_INVALID_ARG, "invalid sizes or parameters for the host call")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = torch.empty(size, dtype=torch.uint8, device=dev)
    ws[:256].zero_()
    return ws


def attention_host(q, k, v, cfg: SparsePRConfig, out: Optional[torch.Tensor] = None, groups: int = 4,
                   ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The call from host tensors (``sparsepr_attention_host``): heads in ``groups`` groups,
    the copies of neighbouring groups overlapping each group's compute.  q, k, v and out
    live in page-locked host memory for the overlap; out is complete once the current
    stream is (``torch.cuda.current_stream().synchronize()``)."""
    for t in (q, k, v):
        if t.is_cuda or not t.is_contiguous():
            raise SparsePRError(ERR_INVALID_ARG, "attention_host takes contiguous host tensors")
    bt, h, n, d = q.shape
    ws = host_workspace(q, cfg, groups) if ws is None else ws
    o = torch.empty(q.shape, dtype=q.dtype, pin_memory=True) if out is None else out
    dev = ws.device
    copy = _COPY_STREAMS.get(dev.index)
    if copy is None:
        copy = _COPY_STREAMS[dev.index] = torch.cuda.Stream(device=dev)
    _call("sparsepr_attention_host", _p(q), _p(k), _p(v), _dtype_code(q), bt, h, n, d, ctypes.byref(cfg.c()),
          _p(o), groups, _p(ws), ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream),
          ctypes.c_void_p(copy.cuda_stream))
    return o
