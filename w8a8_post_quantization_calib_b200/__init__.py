"""SmoothQuant W8A8 linear layer for NVIDIA B200 (sm_100a).

Thin Python binding of ``libsq.so`` (the CUDA kernels behind the C ABI of
``include/sq.h``).  The functions here only marshal arguments: they take
CUDA ``torch.Tensor`` objects (PyTorch supplies device memory and streams),
pass raw pointers and sizes to the library, and raise ``SQError`` on a
non-OK status.  Every step of the layer runs in the library's kernels; there
is no CPU path.  Importing this package on a machine without the built
library raises ``ImportError`` (build it with
``python -m w8a8_post_quantization_calib_b200.build``).

Names follow the C ABI: ``calib_absmax``, ``smooth_scales``,
``quant_weight``, ``smooth_quant_act``, ``linear_w8a8`` (+ ``gemm_s32``,
``quant_weight_gateup``, ``rmsnorm_quant``, ``linear_w8a8_gateup_silu``,
``gemm_f16_ref``, ``sse_f16``, ``alpha_search``) and the FP8 (E4M3) variant
``smooth_scales_fp8``, ``quant_weight_fp8``, ``smooth_quant_act_fp8``,
``linear_fp8`` (codes are uint8 tensors holding E4M3 bit patterns), and the
robust calibration statistics ``calib_quantile``,
``calib_batchmax_accumulate``, ``calib_mean_of_max``, and the cross-layer fold
and fp16 scale storage ``quant_weight_fold``, ``quant_weight_gateup_fold``,
``scales_to_f16``, ``scales_from_f16``, ``linear_w8a8_f16scales``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsq.so")

SQ_F32, SQ_F16, SQ_BF16 = 0, 1, 2
ACT_STATIC, ACT_PER_TOKEN = 0, 1
ALPHA_GRID = (0.25, 0.5, 0.75, 1.0)

_STATUS = {0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_UNSUPPORTED", 3: "SQ_ERR_MISALIGNED",
           4: "SQ_ERR_CUDA", 5: "SQ_ERR_TIMEOUT", 6: "SQ_ERR_WORKSPACE"}

EXPORTS = (
    "sq_status_string", "sq_last_cuda_error", "sq_set_wait_timeout_ns", "sq_debug_inject", "sq_sync_status",
    "sq_calib_absmax", "sq_smooth_scales", "sq_quant_weight", "sq_quant_weight_gateup",
    "sq_smooth_quant_act", "sq_rmsnorm_quant", "sq_rmsnorm_absmax", "sq_linear_workspace_size", "sq_linear_w8a8",
    "sq_linear_w8a8_noalloc", "sq_linear_w8a8_noalloc_max_elems",
    "sq_gemm_s32", "sq_linear_w8a8_gateup_silu", "sq_gemm_f16_ref", "sq_sse_f16",
    "sq_alpha_search_workspace_size", "sq_alpha_search",
    "sq_smooth_scales_fp8", "sq_quant_weight_fp8", "sq_smooth_quant_act_fp8", "sq_linear_fp8",
    "sq_calib_quantile_workspace_size", "sq_calib_quantile", "sq_calib_batchmax_accumulate", "sq_calib_mean_of_max",
    "sq_quant_weight_fold", "sq_quant_weight_gateup_fold", "sq_scales_to_f16", "sq_scales_from_f16",
    "sq_linear_w8a8_f16scales", "sq_linear_w8a8_gateup_silu_absmax",
)


class SQError(RuntimeError):
    def __init__(self, func: str, status: int):
        self.status = status
        extra = ""
        if status == 4:
            extra = f" (cudaError {_lib.sq_last_cuda_error()})"
        super().__init__(f"{func}: {_STATUS.get(status, status)}{extra}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m w8a8_post_quantization_calib_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I, F, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "sq_status_string": (ctypes.c_char_p, [I]),
        "sq_last_cuda_error": (I, []),
        "sq_set_wait_timeout_ns": (None, [ctypes.c_ulonglong]),
        "sq_debug_inject": (None, [I]),
        "sq_sync_status": (I, [P]),
        "sq_calib_absmax": (I, [P, I, I64, I64, I64, P, P]),
        "sq_smooth_scales": (I, [P, P, I64, F, P, P, P]),
        "sq_quant_weight": (I, [P, I, I64, I64, P, P, P, P]),
        "sq_quant_weight_gateup": (I, [P, P, I, I64, I64, P, P, P, P]),
        "sq_smooth_quant_act": (I, [P, I, I64, I64, P, I, P, P, P]),
        "sq_rmsnorm_quant": (I, [P, I, I64, I64, P, P, F, P, P, P, P]),
        "sq_rmsnorm_absmax": (I, [P, I, I64, I64, P, F, P, P]),
        "sq_linear_workspace_size": (SZ, [I64, I64, I64]),
        "sq_linear_w8a8": (I, [P, P, I64, I64, I64, P, I, P, P, I, P, P, SZ, P]),
        "sq_linear_w8a8_noalloc": (I, [P, P, I64, I64, I64, P, I, P, P, I, P, P]),
        "sq_linear_w8a8_noalloc_max_elems": (SZ, []),
        "sq_gemm_s32": (I, [P, P, I64, I64, I64, P, P]),
        "sq_linear_w8a8_gateup_silu": (I, [P, P, I64, I64, I64, P, I, P, P, P, P, P, P]),
        "sq_gemm_f16_ref": (I, [P, P, I64, I64, I64, P, P]),
        "sq_sse_f16": (I, [P, P, I64, P, P]),
        "sq_alpha_search_workspace_size": (SZ, [I64, I64, I64, I]),
        "sq_alpha_search": (I, [P, P, I64, I64, I64, P, P, P, I, P, SZ, P, P, P]),
        "sq_smooth_scales_fp8": (I, [P, P, I64, F, P, P, P]),
        "sq_quant_weight_fp8": (I, [P, I, I64, I64, P, P, P, P]),
        "sq_smooth_quant_act_fp8": (I, [P, I, I64, I64, P, I, P, P, P]),
        "sq_linear_fp8": (I, [P, P, I64, I64, I64, P, I, P, P, I, P, P]),
        "sq_calib_quantile_workspace_size": (SZ, [I64]),
        "sq_calib_quantile": (I, [P, I, I64, I64, I64, ctypes.c_double, P, P, SZ, P]),
        "sq_calib_batchmax_accumulate": (I, [P, I, I64, I64, I64, P, P, P]),
        "sq_calib_mean_of_max": (I, [P, I64, I64, P, P]),
        "sq_quant_weight_fold": (I, [P, I, I64, I64, P, P, P, P, P]),
        "sq_quant_weight_gateup_fold": (I, [P, P, I, I64, I64, P, P, P, P, P]),
        "sq_scales_to_f16": (I, [P, I64, P, P]),
        "sq_scales_from_f16": (I, [P, I64, P, P]),
        "sq_linear_w8a8_f16scales": (I, [P, P, I64, I64, I64, P, I, P, P, I, P, P, SZ, P]),
        "sq_linear_w8a8_gateup_silu_absmax": (I, [P, P, I64, I64, I64, P, I, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


# ---------------------------------------------------------------- marshalling
_DT = {torch.float32: SQ_F32, torch.float16: SQ_F16, torch.bfloat16: SQ_BF16}


def _dt(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(name: str, status: int) -> None:
    if status != 0:
        raise SQError(name, status)


# ---------------------------------------------------------------- the C ABI
def set_wait_timeout_ns(ns: int) -> None:
    _lib.sq_set_wait_timeout_ns(int(ns))


def sync_status(stream=None) -> int:
    """Synchronise the stream; returns the status (0 = OK, 5 = a barrier wait timed out)."""
    return int(_lib.sq_sync_status(_stream(stream)))


def calib_absmax(x: torch.Tensor, absmax: torch.Tensor, rows=None, cols=None, ld=None, stream=None) -> None:
    """absmax[j] = max(absmax[j], max_r |x[r, j]|) for a 2-D x (running max)."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows, cols]")
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[1] if cols is None else cols
    ld = x.stride(0) if ld is None else ld
    if not x.is_cuda:
        raise TypeError("x must be a CUDA tensor")
    _check("sq_calib_absmax", _lib.sq_calib_absmax(x.data_ptr(), _dt(x), rows, cols, ld,
                                                    _dev(absmax, "absmax", torch.float32), _stream(stream)))


def smooth_scales(act_max, w_max, alpha: float, s, a_static=None, stream=None) -> None:
    K = act_max.numel()
    _check("sq_smooth_scales", _lib.sq_smooth_scales(
        _dev(act_max, "act_max", torch.float32), _dev(w_max, "w_max", torch.float32), K, float(alpha),
        _dev(s, "s", torch.float32), _dev(a_static, "a_static", torch.float32), _stream(stream)))


def quant_weight(w, s, wq, w_scale, stream=None) -> None:
    N, K = w.shape
    _check("sq_quant_weight", _lib.sq_quant_weight(
        _dev(w, "w"), _dt(w), N, K, _dev(s, "s", torch.float32), _dev(wq, "wq", torch.int8),
        _dev(w_scale, "w_scale", torch.float32), _stream(stream)))


def quant_weight_gateup(w_gate, w_up, s, wq_gu, w_scale_gu, stream=None) -> None:
    N_h, K = w_gate.shape
    if w_up.shape != w_gate.shape or w_up.dtype != w_gate.dtype:
        raise ValueError("w_gate and w_up must match")
    _check("sq_quant_weight_gateup", _lib.sq_quant_weight_gateup(
        _dev(w_gate, "w_gate"), _dev(w_up, "w_up"), _dt(w_gate), N_h, K, _dev(s, "s", torch.float32),
        _dev(wq_gu, "wq_gu", torch.int8), _dev(w_scale_gu, "w_scale_gu", torch.float32), _stream(stream)))


def smooth_quant_act(x, s, mode: int, a_scale, xq, stream=None) -> None:
    M, K = x.shape
    _check("sq_smooth_quant_act", _lib.sq_smooth_quant_act(
        _dev(x, "x"), _dt(x), M, K, _dev(s, "s", torch.float32), int(mode),
        _dev(a_scale, "a_scale", torch.float32), _dev(xq, "xq", torch.int8), _stream(stream)))


def rmsnorm_quant(x, gamma, s, eps: float, a_scale, xq, rstd=None, stream=None) -> None:
    M, d = x.shape
    _check("sq_rmsnorm_quant", _lib.sq_rmsnorm_quant(
        _dev(x, "x"), _dt(x), M, d, _dev(gamma, "gamma", torch.float32), _dev(s, "s", torch.float32),
        float(eps), _dev(a_scale, "a_scale", torch.float32), _dev(xq, "xq", torch.int8),
        _dev(rstd, "rstd", torch.float32), _stream(stream)))


def rmsnorm_absmax(x, gamma, eps: float, absmax, stream=None) -> None:
    """absmax[j] = max(absmax[j], max_m |RMSNorm(x)[m, j] * gamma[j]|) (running max)."""
    M, d = x.shape
    _check("sq_rmsnorm_absmax", _lib.sq_rmsnorm_absmax(
        _dev(x, "x"), _dt(x), M, d, _dev(gamma, "gamma", torch.float32), float(eps),
        _dev(absmax, "absmax", torch.float32), _stream(stream)))


def linear_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.sq_linear_workspace_size(M, N, K))


def linear_w8a8(xq, wq, a_scale, mode: int, w_scale, y, bias=None, workspace=None, stream=None) -> None:
    M, K = xq.shape
    N = wq.shape[0]
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("sq_linear_w8a8", _lib.sq_linear_w8a8(
        _dev(xq, "xq", torch.int8), _dev(wq, "wq", torch.int8), M, N, K,
        _dev(a_scale, "a_scale", torch.float32), int(mode), _dev(w_scale, "w_scale", torch.float32),
        _dev(bias, "bias", y.dtype) if bias is not None else None, _dt(y), _dev(y, "y"),
        ws_ptr, ws_bytes, _stream(stream)))


def linear_w8a8_noalloc(xq, wq, a_scale, mode: int, w_scale, y, bias=None, stream=None) -> None:
    """linear_w8a8 without a workspace, for callers that cannot allocate device memory.

    The small-M split-K path uses a fixed array inside the library instead
    (calls on one device share it: do not overlap them on the GPU).
    """
    M, K = xq.shape
    N = wq.shape[0]
    _check("sq_linear_w8a8_noalloc", _lib.sq_linear_w8a8_noalloc(
        _dev(xq, "xq", torch.int8), _dev(wq, "wq", torch.int8), M, N, K,
        _dev(a_scale, "a_scale", torch.float32), int(mode), _dev(w_scale, "w_scale", torch.float32),
        _dev(bias, "bias", y.dtype) if bias is not None else None, _dt(y), _dev(y, "y"), _stream(stream)))


def gemm_s32(xq, wq, acc, stream=None) -> None:
    M, K = xq.shape
    N = wq.shape[0]
    _check("sq_gemm_s32", _lib.sq_gemm_s32(
        _dev(xq, "xq", torch.int8), _dev(wq, "wq", torch.int8), M, N, K, _dev(acc, "acc", torch.int32),
        _stream(stream)))


def linear_w8a8_gateup_silu(xq, wq_gu, a_scale, mode: int, w_scale_gu, h=None, s2=None, a2=None, hq=None,
                            stream=None) -> None:
    M, K = xq.shape
    N_h = wq_gu.shape[0] // 2
    _check("sq_linear_w8a8_gateup_silu", _lib.sq_linear_w8a8_gateup_silu(
        _dev(xq, "xq", torch.int8), _dev(wq_gu, "wq_gu", torch.int8), M, N_h, K,
        _dev(a_scale, "a_scale", torch.float32), int(mode), _dev(w_scale_gu, "w_scale_gu", torch.float32),
        _dev(h, "h", torch.bfloat16) if h is not None else None,
        _dev(s2, "s2", torch.float32) if s2 is not None else None,
        _dev(a2, "a2", torch.float32) if a2 is not None else None,
        _dev(hq, "hq", torch.int8) if hq is not None else None, _stream(stream)))


def linear_w8a8_gateup_silu_absmax(xq, wq_gu, a_scale, mode: int, w_scale_gu, h_absmax, stream=None) -> None:
    """h_absmax[c] = max(h_absmax[c], max_m |h[m, c]|) for h = silu(g) * u of the gate/up GEMM; h is not written."""
    M, K = xq.shape
    N_h = wq_gu.shape[0] // 2
    _check("sq_linear_w8a8_gateup_silu_absmax", _lib.sq_linear_w8a8_gateup_silu_absmax(
        _dev(xq, "xq", torch.int8), _dev(wq_gu, "wq_gu", torch.int8), M, N_h, K,
        _dev(a_scale, "a_scale", torch.float32), int(mode), _dev(w_scale_gu, "w_scale_gu", torch.float32),
        _dev(h_absmax, "h_absmax", torch.float32), _stream(stream)))


def gemm_f16_ref(x, w, y, stream=None) -> None:
    M, K = x.shape
    N = w.shape[0]
    _check("sq_gemm_f16_ref", _lib.sq_gemm_f16_ref(
        _dev(x, "x", torch.float16), _dev(w, "w", torch.float16), M, N, K, _dev(y, "y", torch.float16),
        _stream(stream)))


def sse_f16(y, y_ref, sse, stream=None) -> None:
    _check("sq_sse_f16", _lib.sq_sse_f16(
        _dev(y, "y", torch.float16), _dev(y_ref, "y_ref", torch.float16), y.numel(),
        _dev(sse, "sse", torch.float64), _stream(stream)))


def alpha_search_workspace_size(M_held: int, N: int, K: int, n_alpha: int) -> int:
    return int(_lib.sq_alpha_search_workspace_size(M_held, N, K, n_alpha))


def alpha_search(x_held, w, act_max, w_max, workspace, alphas=ALPHA_GRID, stream=None):
    """Per-layer alpha search; returns (best_alpha, [mse per alpha]).  Synchronises the stream."""
    M_h, K = x_held.shape
    N = w.shape[0]
    n = len(alphas)
    al = (ctypes.c_float * n)(*[float(a) for a in alphas])
    best = ctypes.c_float(0.0)
    mse = (ctypes.c_double * n)()
    _check("sq_alpha_search", _lib.sq_alpha_search(
        _dev(x_held, "x_held", torch.float16), _dev(w, "w", torch.float16), M_h, N, K,
        _dev(act_max, "act_max", torch.float32), _dev(w_max, "w_max", torch.float32), al, n,
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        ctypes.byref(best), mse, _stream(stream)))
    return float(best.value), [float(v) for v in mse]


# ---------------------------------------------------------------- FP8 (E4M3) variant
def smooth_scales_fp8(act_max, w_max, alpha: float, s, a_static=None, stream=None) -> None:
    K = act_max.numel()
    _check("sq_smooth_scales_fp8", _lib.sq_smooth_scales_fp8(
        _dev(act_max, "act_max", torch.float32), _dev(w_max, "w_max", torch.float32), K, float(alpha),
        _dev(s, "s", torch.float32), _dev(a_static, "a_static", torch.float32), _stream(stream)))


def quant_weight_fp8(w, s, wq8, w_scale, stream=None) -> None:
    N, K = w.shape
    _check("sq_quant_weight_fp8", _lib.sq_quant_weight_fp8(
        _dev(w, "w"), _dt(w), N, K, _dev(s, "s", torch.float32), _dev(wq8, "wq8", torch.uint8),
        _dev(w_scale, "w_scale", torch.float32), _stream(stream)))


def smooth_quant_act_fp8(x, s, mode: int, a_scale, xq8, stream=None) -> None:
    M, K = x.shape
    _check("sq_smooth_quant_act_fp8", _lib.sq_smooth_quant_act_fp8(
        _dev(x, "x"), _dt(x), M, K, _dev(s, "s", torch.float32), int(mode),
        _dev(a_scale, "a_scale", torch.float32), _dev(xq8, "xq8", torch.uint8), _stream(stream)))


def linear_fp8(xq8, wq8, a_scale, mode: int, w_scale, y, bias=None, stream=None) -> None:
    M, K = xq8.shape
    N = wq8.shape[0]
    _check("sq_linear_fp8", _lib.sq_linear_fp8(
        _dev(xq8, "xq8", torch.uint8), _dev(wq8, "wq8", torch.uint8), M, N, K,
        _dev(a_scale, "a_scale", torch.float32), int(mode), _dev(w_scale, "w_scale", torch.float32),
        _dev(bias, "bias", y.dtype) if bias is not None else None, _dt(y), _dev(y, "y"), _stream(stream)))


# ---------------------------------------------------------------- robust calibration statistics
def calib_quantile_workspace_size(cols: int) -> int:
    return int(_lib.sq_calib_quantile_workspace_size(cols))


def calib_quantile(x: torch.Tensor, p: float, out: torch.Tensor, workspace: torch.Tensor, rows=None, cols=None,
                   ld=None, stream=None) -> None:
    """out[j] = nearest-rank p-quantile of |x[:, j]| over the rows of a 2-D x."""
    if x.dim() != 2 or x.stride(1) != 1 or not x.is_cuda:
        raise ValueError("x must be a 2-D CUDA tensor with contiguous rows")
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[1] if cols is None else cols
    ld = x.stride(0) if ld is None else ld
    _check("sq_calib_quantile", _lib.sq_calib_quantile(
        x.data_ptr(), _dt(x), rows, cols, ld, float(p), _dev(out, "out", torch.float32),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def calib_batchmax_accumulate(x: torch.Tensor, batch_max: torch.Tensor, sum_max: torch.Tensor, stream=None) -> None:
    """sum_max[j] += max_r |x[r, j]| (fp64, one calibration batch per call); batch_max is zeroed scratch."""
    if x.dim() != 2 or x.stride(1) != 1 or not x.is_cuda:
        raise ValueError("x must be a 2-D CUDA tensor with contiguous rows")
    _check("sq_calib_batchmax_accumulate", _lib.sq_calib_batchmax_accumulate(
        x.data_ptr(), _dt(x), x.shape[0], x.shape[1], x.stride(0), _dev(batch_max, "batch_max", torch.float32),
        _dev(sum_max, "sum_max", torch.float64), _stream(stream)))


def calib_mean_of_max(sum_max: torch.Tensor, n_batches: int, out: torch.Tensor, stream=None) -> None:
    _check("sq_calib_mean_of_max", _lib.sq_calib_mean_of_max(
        _dev(sum_max, "sum_max", torch.float64), sum_max.numel(), int(n_batches), _dev(out, "out", torch.float32),
        _stream(stream)))


# ---------------------------------------------------------------- cross-layer fold, fp16 scale storage
def quant_weight_fold(w, s, s_next, wq, w_scale, stream=None) -> None:
    """Per-row INT8 transform of a previous layer's weight with 1/s_next folded into its output rows."""
    N, K = w.shape
    _check("sq_quant_weight_fold", _lib.sq_quant_weight_fold(
        _dev(w, "w"), _dt(w), N, K, _dev(s, "s", torch.float32), _dev(s_next, "s_next", torch.float32),
        _dev(wq, "wq", torch.int8), _dev(w_scale, "w_scale", torch.float32), _stream(stream)))


def quant_weight_gateup_fold(w_gate, w_up, s, s_next, wq_gu, w_scale_gu, stream=None) -> None:
    N_h, K = w_gate.shape
    if w_up.shape != w_gate.shape or w_up.dtype != w_gate.dtype:
        raise ValueError("w_gate and w_up must match")
    _check("sq_quant_weight_gateup_fold", _lib.sq_quant_weight_gateup_fold(
        _dev(w_gate, "w_gate"), _dev(w_up, "w_up"), _dt(w_gate), N_h, K, _dev(s, "s", torch.float32),
        _dev(s_next, "s_next", torch.float32), _dev(wq_gu, "wq_gu", torch.int8),
        _dev(w_scale_gu, "w_scale_gu", torch.float32), _stream(stream)))


def scales_to_f16(x, out, stream=None) -> None:
    """fp32 scales -> fp16 storage (round to nearest even); out: float16 tensor."""
    _check("sq_scales_to_f16", _lib.sq_scales_to_f16(
        _dev(x, "x", torch.float32), x.numel(), _dev(out, "out", torch.float16), _stream(stream)))


def scales_from_f16(x, out, stream=None) -> None:
    _check("sq_scales_from_f16", _lib.sq_scales_from_f16(
        _dev(x, "x", torch.float16), x.numel(), _dev(out, "out", torch.float32), _stream(stream)))


def linear_w8a8_f16scales(xq, wq, a_scale, mode: int, w_scale, y, bias=None, workspace=None, stream=None) -> None:
    """linear_w8a8 with a_scale and w_scale stored as float16."""
    M, K = xq.shape
    N = wq.shape[0]
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("sq_linear_w8a8_f16scales", _lib.sq_linear_w8a8_f16scales(
        _dev(xq, "xq", torch.int8), _dev(wq, "wq", torch.int8), M, N, K,
        _dev(a_scale, "a_scale", torch.float16), int(mode), _dev(w_scale, "w_scale", torch.float16),
        _dev(bias, "bias", y.dtype) if bias is not None else None, _dt(y), _dev(y, "y"),
        ws_ptr, ws_bytes, _stream(stream)))
