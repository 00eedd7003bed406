"""CPU oracle for the SmoothQuant W8A8 linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference`` arm) may import
this package.  The product package never imports it, and it never imports the
product package: the two share no code.  Inputs come from ``synth`` (seeded
generators only, none of the method's arithmetic).

The scalar work lives in ``sq_oracle.c`` (plain C, fp32 operations written out
one by one, ``-ffp-contract=off``); this module compiles it, wraps it with
ctypes/numpy and adds the fp64 numpy checks and the per-workload pipelines.

Sources (the five pages on SmoothQuant):
  [KWKR]  kwkr.cn blog on SmoothQuant W8A8 (sections 1.2, 2.1-2.3, 3.1-3.3, 5.2)
  [TBR8]  tbr8.org article on activation outliers (PyTorch toy example)
  [PWWT]  pwwt.cn "SmoothQuant技术解析：LLM模型INT8无损量化实践" (2.2, 3.1)
  [AIU]   aiunderstanding.org "SmoothQuant 和激活量化" (technical insight)
  [ADR10] blog.yoooo.fun "010. SmoothQuant Integration" (context, key design
          points 1-6, consequences)

Parity pins (tests/test_oracle_pins.py; tests/golden/ fixtures):
  f16/bf16 conversions  -- exhaustive / random vs numpy and torch CPU casts
  quant rule            -- [KWKR] 1.2 worked numbers (golden), RNE ties
  calib_absmax          -- numpy reduction, running-max == concatenated max,
                           outlier channel reads back exactly 100.0
  calib_quantile        -- p = 1 equals calib_absmax; numpy's inverted-CDF
                           quantile (the nearest-rank definition); a planted
                           outlier token moves the max but not the 99.9 %
                           quantile ([KWKR] 3.1)
  calib_mean_of_max     -- equal batch maxima give the max; constructed
                           per-batch maxima give their exact mean; bounded by
                           the smallest and largest batch maximum
  e4m3_decode / encode  -- all 256 codes and in-range values (ties included)
                           against torch's float8_e4m3fn casts; saturation
                           to +-448 beyond (torch gives NaN there)
  fp8 quantisers        -- the row maximum maps to +-448; every code within
                           half an E4M3 spacing of its value
  static_scale_fp8      -- brute force over every smoothed calibration value
  gemm_fp8_f64          -- exact: equals the int64 matmul of the codes'
                           values scaled by 2^9
  fold_into_previous    -- fp64 identity (X Wp'^T)(W diag(s))^T == (X Wp^T) W^T,
                           also through the gated form silu(g) * u
  scales_fp16           -- numpy's float16 round trip
  smooth_scales         -- alpha = 0.5 / 1 / 0 closed forms, clamp at 1e-5
  static_scale          -- brute force over every smoothed calibration value
                           (bit-exact: fl() is monotone)
  quant_weight          -- row argmax -> +-127, |w' - q*scale| <= scale/2
  smooth_quant_act      -- same bounds, static and per-token
  gemm_s32              -- numpy int64 matmul (ragged shapes)
  dequant               -- fp64 product within one fp32 rounding + one output
                           rounding
  dequant_f32           -- hand-computed values that each canonical rounding
                           decides ((float)acc, fl(a_m * w_n), the product),
                           per-token rows with distinct scales; fp64 bound;
                           equal to dequant(..., F32, bias=None)
  rmsnorm_quant         -- fp64 unfused RMSNorm then x/s, within rounding
  rmsnorm_absmax        -- fp64 unfused RMSNorm column max, within rounding
  silu_mul_bf16         -- math.exp closed form on a grid reaching the
                           overflow range of exp (|g| up to 100); silu(0) = 0,
                           silu(g) -> g, silu(-g) -> 0
  mse_f16, gemm_f16_ref -- numpy fp64 mean / matmul
  identity              -- fp64 XW^T == (X diag(s)^-1)(W diag(s))^T, 1e-9;
                           smooth_operands on a hand-computed 2x2 case;
                           rel_residual on a hand value; negative controls
                           (s applied to one operand only) give residuals
                           far above 1e-9
  quality gain          -- [ADR10] consequences: ~10x lower error with
                           smoothing on the outlier layer; not worse on normal
                           activations; smoothing after quantisation gives no
                           gain ([KWKR] 5.2).  The exact factor is
                           "parity unpinned" (the page gives only "about an
                           order of magnitude"); the test bounds it below.
  alpha_search          -- argmin over the grid equals an fp64 numpy
                           re-evaluation (fp64 dequant product) whose MSEs
                           agree within 1e-4 relative; the chosen MSE is <=
                           both extremes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libsq_oracle.so")
_lock = threading.Lock()
_lib = None

F32, F16, BF16 = 0, 1, 2
STATIC, PER_TOKEN = 0, 1
ALPHA_GRID = (0.25, 0.5, 0.75, 1.0)   # [ADR10] key design point 2
ALPHA_DEFAULT = 0.5                    # [KWKR] 2.2, [AIU], [ADR10] key design point 2
CLAMP_MIN = 1e-5                       # [TBR8] s.clamp(min=1e-5)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile sq_oracle.c into oracle/_build/libsq_oracle.so (gcc, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_SO)
            and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
        return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.oracle_f16_to_f32.restype = ctypes.c_float
            L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_f32.restype = ctypes.c_float
            L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.oracle_f32_to_f16.restype = ctypes.c_uint16
            L.oracle_f32_to_f16.argtypes = [ctypes.c_float]
            L.oracle_f32_to_bf16.restype = ctypes.c_uint16
            L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
            L.oracle_recip.restype = ctypes.c_float
            L.oracle_recip.argtypes = [ctypes.c_float]
            L.oracle_quant.restype = ctypes.c_int8
            L.oracle_quant.argtypes = [ctypes.c_float]
            L.oracle_calib_absmax.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, _P]
            L.oracle_smooth_scales.argtypes = [_P, _P, _I64, ctypes.c_float, _P]
            L.oracle_static_scale.restype = ctypes.c_float
            L.oracle_static_scale.argtypes = [_P, _P, _I64]
            L.oracle_quant_weight.argtypes = [_P, ctypes.c_int, _I64, _I64, _P, _P, _P]
            L.oracle_smooth_quant_act.argtypes = [_P, ctypes.c_int, _I64, _I64, _P, ctypes.c_int, _P, _P]
            L.oracle_gemm_s32.argtypes = [_P, _P, _I64, _I64, _I64, _P]
            L.oracle_dequant.argtypes = [_P, _I64, _I64, _P, ctypes.c_int, _P, _P, ctypes.c_int, _P]
            L.oracle_dequant_f32.argtypes = [_P, _I64, _I64, _P, ctypes.c_int, _P, _P]
            L.oracle_rmsnorm_quant.argtypes = [_P, ctypes.c_int, _I64, _I64, _P, _P, ctypes.c_float,
                                               _P, _P, _P, _P]
            L.oracle_silu_mul_bf16.argtypes = [_P, _P, _I64, _P]
            L.oracle_rmsnorm_absmax.argtypes = [_P, ctypes.c_int, _I64, _I64, _P, ctypes.c_float, _P]
            L.oracle_mse_f16.restype = ctypes.c_double
            L.oracle_mse_f16.argtypes = [_P, _P, _I64]
            L.oracle_gemm_f16_ref.argtypes = [_P, _P, _I64, _I64, _I64, _P]
            L.oracle_to_f32_array.argtypes = [_P, ctypes.c_int, _I64, _P]
            L.oracle_from_f32_array.argtypes = [_P, _I64, ctypes.c_int, _P]
            _lib = L
    return _lib


# --------------------------------------------------------------------------
# numpy helpers.  16-bit tensors travel as uint16 bit patterns (bf16 has no
# numpy dtype); fp16 arrays are accepted and viewed as uint16.
# --------------------------------------------------------------------------

def _dtcode(a: np.ndarray, dt: int | None) -> tuple[np.ndarray, int]:
    if dt is None:
        if a.dtype == np.float32:
            dt = F32
        elif a.dtype == np.float16:
            dt = F16
        else:
            raise TypeError("bf16 data is passed as uint16 with dt=BF16")
    if dt == F32:
        a = np.ascontiguousarray(a, dtype=np.float32)
    else:
        a = np.ascontiguousarray(a).view(np.uint16)
    return a, dt


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def to_f32(a: np.ndarray, dt: int) -> np.ndarray:
    """Widen a 16-bit bit-pattern array (or an fp32 array) to fp32, exactly."""
    if dt == F32:
        return np.array(a, dtype=np.float32)
    bits = np.ascontiguousarray(a).view(np.uint16)
    out = np.empty(bits.shape, np.float32)
    lib().oracle_to_f32_array(_ptr(bits), dt, bits.size, _ptr(out))
    return out


def from_f32(a: np.ndarray, dt: int) -> np.ndarray:
    """Round fp32 values to dt (RNE); 16-bit results are uint16 bit patterns."""
    a = np.ascontiguousarray(a, np.float32)
    if dt == F32:
        return a.copy()
    out = np.empty(a.shape, np.uint16)
    lib().oracle_from_f32_array(_ptr(a), a.size, dt, _ptr(out))
    return out


def quant(v: float) -> int:
    """[KWKR] 1.2: x_q = round(x / s); RNE, saturate to +-127."""
    return int(lib().oracle_quant(float(v)))


def recip(v: float) -> float:
    return float(lib().oracle_recip(float(v)))


def calib_absmax(x: np.ndarray, dt: int | None = None, absmax: np.ndarray | None = None) -> np.ndarray:
    """a1/a2 -- running per-column max|x| ([KWKR] 3.1; [ADR10] add_batch)."""
    x, dt = _dtcode(x, dt)
    rows, cols = x.shape
    out = np.zeros(cols, np.float32) if absmax is None else absmax
    assert out.dtype == np.float32 and out.flags.c_contiguous
    lib().oracle_calib_absmax(_ptr(x), dt, rows, cols, cols, _ptr(out))
    return out


def quantile_rank(p: float, count: int) -> int:
    """1-based nearest rank of the p-quantile among `count` values: k = ceil(p * count)
    (the product taken in fp64), at least 1 and at most count."""
    import math
    if not (0.0 < p <= 1.0) or count < 1:
        raise ValueError("need 0 < p <= 1 and at least one value")
    return min(count, max(1, math.ceil(float(p) * float(count))))


def calib_quantile(batches, p: float, dt: int | None = None) -> np.ndarray:
    """Robust calibration statistic, [KWKR] 3.1: a quantile of |X_j| over all the
    calibration tokens (the page names 99.9 %) in place of the max, so that one
    sample with an abnormally large activation does not set the channel's s.

    Per channel j the p-quantile by nearest rank: with the T values |x_tj|
    sorted ascending, the k-th smallest, k = quantile_rank(p, T).  It is one
    of the data values (widened exactly to fp32); p = 1 gives the max."""
    cols = [np.abs(to_f32(*_dtcode(b, dt))) for b in batches]
    a = np.concatenate(cols, axis=0)                       # [T, K]
    k = quantile_rank(p, a.shape[0])
    return np.sort(a, axis=0)[k - 1].astype(np.float32)


def calib_mean_of_max(batches, dt: int | None = None) -> np.ndarray:
    """Robust calibration statistic, [KWKR] 3.1: the mean over calibration
    samples of each sample's max|X_j| (a sample being one calibration batch).
    The per-sample maxima are added in fp64 in sample order, the sum is divided
    by the sample count in fp64 and rounded once to fp32."""
    total = None
    for b in batches:
        m = calib_absmax(b, dt).astype(np.float64)
        total = m if total is None else total + m
    return (total / float(len(batches))).astype(np.float32)


def smooth_scales(act_max: np.ndarray, w_max: np.ndarray, alpha: float = ALPHA_DEFAULT) -> np.ndarray:
    """a3 -- s_j = max|X_j|^a / max|W_j|^(1-a) ([KWKR] 2.2; [AIU]; [ADR10] step 1)."""
    a = np.ascontiguousarray(act_max, np.float32)
    w = np.ascontiguousarray(w_max, np.float32)
    s = np.empty_like(a)
    lib().oracle_smooth_scales(_ptr(a), _ptr(w), len(a), float(alpha), _ptr(s))
    return s


def static_scale(act_max: np.ndarray, s: np.ndarray) -> np.float32:
    """a3 -- closed-form per-tensor scale max_j(act_max_j/s_j)/127 ([ADR10] point 1)."""
    a = np.ascontiguousarray(act_max, np.float32)
    s = np.ascontiguousarray(s, np.float32)
    return np.float32(lib().oracle_static_scale(_ptr(a), _ptr(s), len(a)))


def quant_weight(w: np.ndarray, s: np.ndarray, dt: int | None = None):
    """a4 -- W' = W diag(s), per-row INT8 ([KWKR] 3.2-3.3; [ADR10] step 3)."""
    w, dt = _dtcode(w, dt)
    N, K = w.shape
    s = np.ascontiguousarray(s, np.float32)
    wq = np.empty((N, K), np.int8)
    ws = np.empty(N, np.float32)
    lib().oracle_quant_weight(_ptr(w), dt, N, K, _ptr(s), _ptr(wq), _ptr(ws))
    return wq, ws


def smooth_quant_act(x: np.ndarray, s: np.ndarray, mode: int, a_scale=None, dt: int | None = None):
    """a5/a5' -- x/s then INT8 ([KWKR] 3.2, 5.2: smoothing precedes quantisation).

    static: ``a_scale`` is the per-tensor scale; per-token: returns (xq, a[M]).
    """
    x, dt = _dtcode(x, dt)
    M, K = x.shape
    s = np.ascontiguousarray(s, np.float32)
    xq = np.empty((M, K), np.int8)
    if mode == STATIC:
        a = np.array([a_scale], np.float32).ravel()[:1].copy()
    else:
        a = np.empty(M, np.float32)
    lib().oracle_smooth_quant_act(_ptr(x), dt, M, K, _ptr(s), mode, _ptr(a), _ptr(xq))
    return xq, a


# --------------------------------------------------------------------------
# FP8 (E4M3) variant: the same smoothing in front of an FP8 quantiser ([AIU]:
# smoothing carries over to FP8 on Hopper / Blackwell).  E4M3: 1 sign, 4
# exponent bits (bias 7), 3 mantissa bits, no infinities, code 0x7F / 0xFF
# NaN, largest finite 448.
# --------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) -> fp32 values (exact)."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    v = np.where(c & 0x80, -mag, mag)
    v = np.where((c & 0x7F) == 0x7F, np.nan, v)
    return v.astype(np.float32)


_E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)   # codes 0..126, ascending


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3 codes: round to nearest, ties to the even code (even
    mantissa), magnitudes beyond 448 saturate to +-448 (the finite-saturating
    conversion), NaN -> 0x7F.  The nearest of the 127 non-negative finite
    values is found by search over the ascending table."""
    v = np.asarray(v, np.float32)
    a = np.abs(v).astype(np.float64)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 126)    # first value >= a
    lo = np.clip(hi - 1, 0, 126)
    dlo, dhi = a - _E4M3_POS[lo], _E4M3_POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 126, code)                             # saturate
    code = code.astype(np.int64) | np.where(np.signbit(v), 0x80, 0)
    code = np.where(np.isnan(v), 0x7F, code)
    return code.astype(np.uint8)


def _f32(x):
    return np.asarray(x, np.float32)


def _recip32(v: np.ndarray) -> np.ndarray:
    """fl(1/v), 0 for v = 0 (the reciprocal rule of the INT8 path)."""
    v = _f32(v)
    with np.errstate(divide="ignore"):
        return np.where(v > 0, np.float32(1.0) / np.where(v > 0, v, np.float32(1.0)), np.float32(0.0)).astype(np.float32)


def smooth_quant_act_fp8(x: np.ndarray, s: np.ndarray, mode: int, a_scale=None, dt: int | None = None):
    """x/s, then E4M3 with a per-tensor (static) or per-token scale a = max|x'|/448,
    in the INT8 path's fp32 order: x' = fl(x * fl(1/s_j)); code = e4m3(fl(x' * fl(1/a)))."""
    x, dt = _dtcode(x, dt)
    xf = to_f32(x, dt)
    xs = (xf * _recip32(s)[None, :]).astype(np.float32)
    if mode == STATIC:
        a = _f32([a_scale]).ravel()[:1]
        inv = _recip32(a)[0]
        return e4m3_encode((xs * inv).astype(np.float32)), a
    a = (np.abs(xs).max(axis=1) / np.float32(E4M3_MAX)).astype(np.float32)
    return e4m3_encode((xs * _recip32(a)[:, None]).astype(np.float32)), a


def static_scale_fp8(act_max: np.ndarray, s: np.ndarray) -> np.float32:
    """Closed-form per-tensor scale for E4M3 codes ([ADR10] key design point 1
    with 448 in place of 127): fl(max_j fl(act_max_j * fl(1/s_j)) / 448)."""
    m = (_f32(act_max) * _recip32(s)).astype(np.float32).max()
    return np.float32(np.float32(m) / np.float32(E4M3_MAX))


def quant_weight_fp8(w: np.ndarray, s: np.ndarray, dt: int | None = None):
    """W' = fl(W * s_j), per-row scale fl(max|W'_n| / 448), codes e4m3(fl(W' * fl(1/scale)))."""
    w, dt = _dtcode(w, dt)
    wf = (to_f32(w, dt) * _f32(s)[None, :]).astype(np.float32)
    sc = (np.abs(wf).max(axis=1) / np.float32(E4M3_MAX)).astype(np.float32)
    return e4m3_encode((wf * _recip32(sc)[:, None]).astype(np.float32)), sc


def gemm_fp8_f64(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """acc = dec(xq) . dec(wq)^T in fp64.  Every product of two E4M3 values is a
    multiple of 2^-18 below 2^18, so for K < 2^16 the fp64 sum is exact in any order."""
    return e4m3_decode(xq).astype(np.float64) @ e4m3_decode(wq).astype(np.float64).T


def gemm_s32(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """a6 -- acc = xq . wq^T in exact int32."""
    xq = np.ascontiguousarray(xq, np.int8)
    wq = np.ascontiguousarray(wq, np.int8)
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    lib().oracle_gemm_s32(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc))
    return acc


def dequant(acc: np.ndarray, a_scale: np.ndarray, mode: int, w_scale: np.ndarray,
            out_dt: int, bias: np.ndarray | None = None) -> np.ndarray:
    """a6 epilogue -- fmaf((float)acc, fl(a_m*w_n), bias_n) rounded to out_dt.

    Returns fp32 values (out_dt F32) or uint16 bit patterns (F16/BF16).
    """
    acc = np.ascontiguousarray(acc, np.int32)
    M, N = acc.shape
    a = np.ascontiguousarray(a_scale, np.float32).ravel()
    ws = np.ascontiguousarray(w_scale, np.float32)
    if bias is not None:
        bias, _ = _dtcode(bias, out_dt)
    y = np.empty((M, N), np.float32 if out_dt == F32 else np.uint16)
    lib().oracle_dequant(_ptr(acc), M, N, _ptr(a), mode, _ptr(ws), _ptr(bias), out_dt, _ptr(y))
    return y


def dequant_f32(acc, a_scale, mode, w_scale) -> np.ndarray:
    """a9 -- the a6 epilogue values in fp32, no bias, no output rounding:
    y = fl((float)acc * fl(a_m * w_n)) (the gate and up values of SiLU*mul)."""
    acc = np.ascontiguousarray(acc, np.int32)
    M, N = acc.shape
    a = np.ascontiguousarray(a_scale, np.float32).ravel()
    ws = np.ascontiguousarray(w_scale, np.float32)
    y = np.empty((M, N), np.float32)
    lib().oracle_dequant_f32(_ptr(acc), M, N, _ptr(a), mode, _ptr(ws), _ptr(y))
    return y


def rmsnorm_quant(x, gamma, s, eps, a_static, dt: int | None = None, r_given=None):
    """a8 -- RMSNorm with 1/s folded into gamma, then INT8 ([KWKR] 2.3, 3.2; [AIU]).

    Returns (xq, r) where r[m] = 1/sqrt(mean x^2 + eps) (or ``r_given``).
    """
    x, dt = _dtcode(x, dt)
    M, d = x.shape
    g = np.ascontiguousarray(gamma, np.float32)
    s = np.ascontiguousarray(s, np.float32)
    a = np.array([a_static], np.float32).ravel()[:1].copy()
    rg = None if r_given is None else np.ascontiguousarray(r_given, np.float32)
    xq = np.empty((M, d), np.int8)
    r = np.empty(M, np.float32)
    lib().oracle_rmsnorm_quant(_ptr(x), dt, M, d, _ptr(g), _ptr(s), float(eps), _ptr(a),
                               _ptr(rg), _ptr(xq), _ptr(r))
    return xq, r


def rmsnorm_absmax(x, gamma, eps, dt: int | None = None, absmax: np.ndarray | None = None) -> np.ndarray:
    """Running column max of |RMSNorm(x) * gamma| (the gate/up layer's input statistic)."""
    x, dt = _dtcode(x, dt)
    M, d = x.shape
    g = np.ascontiguousarray(gamma, np.float32)
    out = np.zeros(d, np.float32) if absmax is None else absmax
    lib().oracle_rmsnorm_absmax(_ptr(x), dt, M, d, _ptr(g), float(eps), _ptr(out))
    return out


def silu_mul_bf16(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """a9 -- h = silu(g) * u, rounded to bf16 (uint16 bits)."""
    g = np.ascontiguousarray(g, np.float32)
    u = np.ascontiguousarray(u, np.float32)
    h = np.empty(g.shape, np.uint16)
    lib().oracle_silu_mul_bf16(_ptr(g), _ptr(u), g.size, _ptr(h))
    return h


def mse_f16(y_bits: np.ndarray, yref_bits: np.ndarray) -> float:
    """a7 -- mean((y - y_ref)^2) in fp64 ([ADR10] point 2: output reconstruction error)."""
    y = np.ascontiguousarray(y_bits).view(np.uint16)
    r = np.ascontiguousarray(yref_bits).view(np.uint16)
    return float(lib().oracle_mse_f16(_ptr(y), _ptr(r), y.size))


def gemm_f16_ref(x_bits: np.ndarray, w_bits: np.ndarray) -> np.ndarray:
    """a7 -- unquantised fp16 product, fp64-accumulated, rounded to fp16 (bits)."""
    x = np.ascontiguousarray(x_bits).view(np.uint16)
    w = np.ascontiguousarray(w_bits).view(np.uint16)
    M, K = x.shape
    N, _ = w.shape
    y = np.empty((M, N), np.uint16)
    lib().oracle_gemm_f16_ref(_ptr(x), _ptr(w), M, N, K, _ptr(y))
    return y


# --------------------------------------------------------------------------
# fp64 numpy checks of the mathematics
# --------------------------------------------------------------------------

def smooth_operands(X: np.ndarray, W: np.ndarray, s: np.ndarray):
    """[KWKR] 2.1: the smoothed pair (X diag(s)^-1, W diag(s)) in fp64.

    X is [M,K]; W is [N,K] (out x in), so diag(s) scales its columns: both
    operands are scaled along the shared input-channel index j."""
    X = np.asarray(X, np.float64)
    W = np.asarray(W, np.float64)
    s = np.asarray(s, np.float64)
    return X / s[None, :], W * s[None, :]


def rel_residual(Y: np.ndarray, Ys: np.ndarray) -> float:
    """Relative Frobenius residual ||Y - Ys|| / ||Y|| in fp64."""
    Y = np.asarray(Y, np.float64)
    Ys = np.asarray(Ys, np.float64)
    return float(np.linalg.norm(Y - Ys) / np.linalg.norm(Y))


def identity_residual(X: np.ndarray, W: np.ndarray, s: np.ndarray) -> float:
    """[KWKR] 2.1: Y = X W^T = (X diag(s)^-1)(W diag(s))^T; relative residual in fp64."""
    Xs, Ws = smooth_operands(X, W, s)
    Y = np.asarray(X, np.float64) @ np.asarray(W, np.float64).T
    return rel_residual(Y, Xs @ Ws.T)


# --------------------------------------------------------------------------
# Follow-ups named by [ADR10]: cross-layer folding (Alternative C) and fp16
# storage of the scales (Consequences, storage)
# --------------------------------------------------------------------------

def fold_into_previous(w_prev: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Cross-layer folding: when the smoothed layer's input is a previous
    linear's output (or depends linearly on it, as h = silu(g) * u does on the
    up projection), 1/s_j moves into that layer's output row j,
    W_prev'[j, :] = fl(W_prev[j, :] * fl(1/s_j)), and the runtime x/s step
    disappears.  w_prev: fp32 [K, K_prev] (out x in); returns fp32."""
    w = np.asarray(w_prev, np.float32)
    return (w * _recip32(s)[:, None]).astype(np.float32)


def scales_fp16(*scales):
    """fp16 storage of scales ([ADR10] consequences: per-row weight scale,
    per-tensor activation scale and input scales s in fp16): each fp32 scale
    rounded to the nearest fp16 (RNE) and read back widened exactly to fp32,
    the values every later step then uses."""
    return tuple(to_f32(from_f32(np.asarray(v, np.float32), F16), F16) for v in scales)


# --------------------------------------------------------------------------
# Pipelines (the same sequence of steps the GPU path runs)
# --------------------------------------------------------------------------

@dataclass
class LinearState:
    act_max: np.ndarray
    w_max: np.ndarray
    s: np.ndarray
    a_static: np.float32
    wq: np.ndarray
    w_scale: np.ndarray


def calibrate_and_quantize(calib_batches, W, alpha=ALPHA_DEFAULT, x_dt=None, w_dt=None) -> LinearState:
    """a1 -> a2 -> a3 -> a4 for one linear layer."""
    K = W.shape[1]
    act_max = np.zeros(K, np.float32)
    for xb in calib_batches:
        calib_absmax(xb, x_dt, act_max)
    w_max = calib_absmax(W, w_dt)
    s = smooth_scales(act_max, w_max, alpha)
    a = static_scale(act_max, s)
    wq, ws = quant_weight(W, s, w_dt)
    return LinearState(act_max, w_max, s, a, wq, ws)


def linear_forward(st: LinearState, X, mode: int, out_dt: int, x_dt=None, bias=None):
    """a5/a5' -> a6: returns (xq, a_scale, acc, y)."""
    if mode == STATIC:
        xq, a = smooth_quant_act(X, st.s, STATIC, st.a_static, x_dt)
    else:
        xq, a = smooth_quant_act(X, st.s, PER_TOKEN, None, x_dt)
    acc = gemm_s32(xq, st.wq)
    y = dequant(acc, a, mode, st.w_scale, out_dt, bias)
    return xq, a, acc, y


def w8a8_output_f64(X, W, s, a_mode=STATIC, act_max=None):
    """fp64 value of the dequantised W8A8 product (for the quality checks)."""
    if a_mode == STATIC:
        a = static_scale(act_max, s)
        xq, av = smooth_quant_act(X, s, STATIC, a)
    else:
        xq, av = smooth_quant_act(X, s, PER_TOKEN)
    wq, ws = quant_weight(W, s)
    acc = gemm_s32(xq, wq).astype(np.float64)
    av = av.astype(np.float64)
    am = av[0] if a_mode == STATIC else av[:, None]
    return acc * am * ws.astype(np.float64)[None, :]


def alpha_search(x_held_bits, w_bits, act_max, w_max, grid=ALPHA_GRID, rel_tie=1e-6):
    """a7 -- per-layer alpha grid search ([ADR10] point 2, honest search).

    For each alpha: s -> static a -> weight quant -> held-batch quant -> INT8
    GEMM -> fp16 output; MSE against the unquantised fp16 product.  Ties
    within ``rel_tie`` go to the smaller alpha.  Returns (alpha, mses, y_ref).
    """
    y_ref = gemm_f16_ref(x_held_bits, w_bits)
    mses = []
    for al in grid:
        s = smooth_scales(act_max, w_max, al)
        a = static_scale(act_max, s)
        wq, ws = quant_weight(w_bits, s, F16)
        xq, av = smooth_quant_act(x_held_bits, s, STATIC, a, F16)
        acc = gemm_s32(xq, wq)
        y = dequant(acc, av, STATIC, ws, F16)
        mses.append(mse_f16(y, y_ref))
    best = 0
    for i in range(1, len(grid)):
        if mses[i] < mses[best] * (1.0 - rel_tie):
            best = i
    return grid[best], mses, y_ref
