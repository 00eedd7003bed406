"""Pins of the CPU oracle to facts fixed by the pages and by mathematics.

Every oracle function is checked here against something other than itself:
worked numbers printed on the pages (tests/golden/), closed forms, exact
invariants, library routines for the special cases that reduce to them
(numpy/torch casts, numpy integer matmul), and brute force on small inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import BF16, F16, F32, PER_TOKEN, STATIC


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.abs(a - b) / np.maximum(np.abs(b), 1e-300)


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def test_f16_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.to_f32(bits, F16)
    ref = bits.view(np.float16).astype(np.float32)
    assert np.array_equal(got, ref, equal_nan=True)


def test_f16_encode_matches_numpy():
    g = np.random.default_rng(7)
    vals = [g.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** g.integers(-9, 6, 20000)]
    # exact ties between representable halves, the overflow edge and subnormals
    h = np.arange(0, 0x7c00, 37, dtype=np.uint16).view(np.float16).astype(np.float32)
    nxt = (np.arange(0, 0x7c00, 37, dtype=np.uint16) + 1).view(np.float16).astype(np.float32)
    vals.append(((h.astype(np.float64) + nxt.astype(np.float64)) / 2).astype(np.float32))
    vals.append(np.array([65504, 65519.99, 65520, 65536, 1e9, 6e-8, 3e-8, 2.98e-8, 0.0, -0.0,
                          np.inf, -np.inf], np.float32))
    v = np.concatenate(vals)
    v = np.concatenate([v, -v])
    got = oracle.from_f32(v, F16)
    with np.errstate(over='ignore'):
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_matches_torch_casts():
    g = np.random.default_rng(8)
    v = (g.standard_normal(50000) * 10.0 ** g.integers(-30, 30, 50000)).astype(np.float32)
    bits32 = np.arange(0, 2 ** 32, 2 ** 32 // 40000, dtype=np.uint64).astype(np.uint32)
    finite = bits32.view(np.float32)
    v = np.concatenate([v, finite[np.isfinite(finite)]])
    got = oracle.from_f32(v, BF16)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    bits = np.arange(65536, dtype=np.uint16)
    dec = oracle.to_f32(bits, BF16)
    tref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    assert np.array_equal(dec, tref, equal_nan=True)


# --------------------------------------------------------------------------
# quantisation rule  (kwkr.cn section 1.2)
# --------------------------------------------------------------------------

def test_quant_rule_ties_even_and_symmetric_saturation():
    assert [oracle.quant(v) for v in (0.5, 1.5, 2.5, -0.5, -2.5, 3.5)] == [0, 2, 2, 0, -2, 4]
    assert oracle.quant(126.5) == 126 and oracle.quant(126.51) == 127
    assert oracle.quant(127.49) == 127 and oracle.quant(1e9) == 127
    assert oracle.quant(-127.5) == -127 and oracle.quant(-1e9) == -127   # never -128
    assert oracle.recip(0.0) == 0.0 and oracle.recip(4.0) == 0.25


def test_kwkr_outlier_quant_worked_numbers(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "kwkr_1_2_outlier_quant.json")))
    big, small = spec["cases"]
    # scale 50/127: the bulk [-1, 1] collapses onto a handful of levels
    s = np.float32(big["scale_num"]) / np.float32(big["scale_den"])
    assert abs(float(s) - big["scale_approx"]) < 0.005
    inv = oracle.recip(float(s))
    assert abs(big["x_hi"] * inv - big["scaled_span_approx"]) < 0.1
    xs = np.linspace(big["x_lo"], big["x_hi"], 20001, dtype=np.float32)
    codes = {oracle.quant(float(np.float32(x) * np.float32(inv))) for x in xs}
    assert len(codes) <= big["levels_at_most"] and codes == set(range(-3, 4))
    # scale 1/127: the outlier 50 lands near 6300+ and saturates at 127
    s2 = np.float32(small["scale_num"]) / np.float32(small["scale_den"])
    assert abs(float(s2) - small["scale_approx"]) < 5e-5
    v = np.float32(small["x"]) * np.float32(oracle.recip(float(s2)))
    assert v >= small["unsaturated_at_least"]
    assert oracle.quant(float(v)) == small["code"]
    assert oracle.quant(float(-v)) == -small["code"]


# --------------------------------------------------------------------------
# a1/a2 calibration statistic
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dt", [F32, F16, BF16])
def test_calib_absmax_vs_numpy(dt):
    g = np.random.default_rng(dt)
    batches = [synth.cast(g.standard_normal((r, 77)).astype(np.float32) * 3, dt) for r in (1, 5, 64)]
    run = np.zeros(77, np.float32)
    for b in batches:
        oracle.calib_absmax(b, dt, run)
    allx = np.concatenate([oracle.to_f32(b, dt) for b in batches])
    assert np.array_equal(run, np.abs(allx).max(axis=0))


@pytest.mark.parametrize("dt", [F32, F16, BF16])
def test_calib_quantile_at_one_is_the_max(dt):
    g = np.random.default_rng(40 + dt)
    batches = [synth.cast(g.standard_normal((r, 53)).astype(np.float32) * 4, dt) for r in (7, 30, 1)]
    run = np.zeros(53, np.float32)
    for b in batches:
        oracle.calib_absmax(b, dt, run)
    assert np.array_equal(oracle.calib_quantile(batches, 1.0, dt), run)


@pytest.mark.parametrize("p", [0.999, 0.9, 0.5, 0.013])
def test_calib_quantile_is_numpy_inverted_cdf(p):
    """Nearest rank k = ceil(pT) is numpy's inverted-CDF quantile (the smallest
    value whose empirical CDF reaches p); T = 3001 keeps pT off the integers."""
    g = np.random.default_rng(41)
    batches = [synth.cast(g.standard_normal((r, 40)).astype(np.float32), BF16) for r in (1000, 2000, 1)]
    a = np.abs(np.concatenate([oracle.to_f32(b, BF16) for b in batches]))
    assert a.shape[0] == 3001 and abs(p * 3001 - round(p * 3001)) > 1e-6
    ref = np.quantile(a, p, axis=0, method="inverted_cdf")
    assert np.array_equal(oracle.calib_quantile(batches, p, BF16), ref.astype(np.float32))


def test_calib_quantile_ignores_a_planted_outlier():
    """[KWKR] 3.1: one sample with an abnormally large activation sets the max
    of its channel; the 99.9 % quantile of 2000 tokens (rank 1998) stays with
    the body of the distribution.  Channel 3: 1999 tokens with |x| = t/2000
    (t = 1..1999) and one token at 5000."""
    x = np.zeros((2000, 8), np.float32)
    x[:1999, 3] = np.arange(1, 2000, dtype=np.float32) / 2000
    x[1999, 3] = -5000.0
    batches = [x[:700], x[700:]]
    assert oracle.quantile_rank(0.999, 2000) == 1998
    q = oracle.calib_quantile(batches, 0.999, F32)
    assert q[3] == np.float32(1998) / 2000            # the 1998-th smallest |x|
    assert oracle.calib_absmax(x, F32)[3] == 5000.0
    assert np.all(q[np.arange(8) != 3] == 0.0)


def test_calib_mean_of_max_closed_forms():
    """[KWKR] 3.1 mean of per-sample maxima: batches whose channel maxima are
    1, 2, 3, 4.5 (exact in every format) give 2.625; equal maxima give that max;
    in general the mean lies between the smallest and largest batch maximum."""
    B, K = 4, 6
    peaks = np.array([1.0, 2.0, 3.0, 4.5], np.float32)
    batches = []
    for b in range(B):
        x = np.full((5, K), 0.25, np.float32)
        x[b + 1, 2] = -peaks[b]                     # channel 2: the planted per-batch maximum
        x[0, 4] = 7.0                              # channel 4: the same maximum in every batch
        batches.append(synth.cast(x, BF16))
    m = oracle.calib_mean_of_max(batches, BF16)
    assert m[2] == np.float32(2.625)
    assert m[4] == np.float32(7.0)
    assert m[0] == np.float32(0.25)
    g = np.random.default_rng(42)
    rb = [synth.cast(g.standard_normal((r, 31)).astype(np.float32) * 2, F16) for r in (3, 50, 9, 17)]
    mm = oracle.calib_mean_of_max(rb, F16)
    per = np.stack([oracle.calib_absmax(b, F16) for b in rb])
    assert np.all(mm >= per.min(axis=0)) and np.all(mm <= per.max(axis=0))


def test_toy_outlier_channel_statistic(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "tbr8_toy_layer.json")))
    wl = synth.linear_toy()
    assert wl.K == spec["in_features"] and wl.N == spec["out_features"]
    am = np.zeros(wl.K, np.float32)
    for b in wl.calib:
        oracle.calib_absmax(b, F32, am)
    assert am[spec["outlier_channel"]] == spec["outlier_value"]
    assert np.argmax(am) == spec["outlier_channel"]
    wm = oracle.calib_absmax(wl.w, F32)
    assert np.array_equal(wm, np.abs(wl.w).max(axis=0))      # column max of [out, in]


# --------------------------------------------------------------------------
# a3 smoothing factors and the closed-form static scale
# --------------------------------------------------------------------------

def _stats(K=300, seed=3):
    g = np.random.default_rng(seed)
    a = (np.abs(g.standard_normal(K)) * 10 + 0.01).astype(np.float32)
    a[::37] *= 50
    w = (np.abs(g.standard_normal(K)) * 0.05 + 1e-3).astype(np.float32)
    return a, w


def test_alpha_half_splits_difficulty_evenly():
    """kwkr.cn 2.2: at alpha = 0.5 the smoothed activation and weight column maxima meet at sqrt(a w)."""
    a, w = _stats()
    s = oracle.smooth_scales(a, w, 0.5)
    gm = np.sqrt(a.astype(np.float64) * w.astype(np.float64))
    assert _rel(a / s.astype(np.float64), gm).max() < 1e-6
    assert _rel(w * s.astype(np.float64), gm).max() < 1e-6


def test_alpha_one_and_zero_limits():
    a, w = _stats()
    s1 = oracle.smooth_scales(a, w, 1.0)     # all difficulty to the weights: act/s == 1
    assert _rel(a / s1.astype(np.float64), 1.0).max() < 1e-6
    s0 = oracle.smooth_scales(a, w, 0.0)     # none: s == 1 / w_max, so W' columns peak at 1
    assert _rel(w * s0.astype(np.float64), 1.0).max() < 1e-6


def test_alpha_monotone_transfer():
    """kwkr.cn 2.2: a larger alpha flattens the activation channels and spreads the weights.

    act_j/s_j = (a_j w_j)^(1-alpha) and w_j s_j = (a_j w_j)^alpha, so the
    cross-channel spread of the smoothed activation maxima shrinks with alpha
    while the spread of the smoothed weight maxima grows.
    """
    a, w = _stats()
    act_spread, w_spread = [], []
    for al in (0.0, 0.25, 0.5, 0.75, 1.0):
        s = oracle.smooth_scales(a, w, al).astype(np.float64)
        act_spread.append((a / s).max() / (a / s).min())
        w_spread.append((w * s).max() / (w * s).min())
    assert all(x >= y * (1 - 1e-6) for x, y in zip(act_spread, act_spread[1:]))
    assert all(x <= y * (1 + 1e-6) for x, y in zip(w_spread, w_spread[1:]))
    assert abs(act_spread[-1] - 1.0) < 1e-5 and abs(w_spread[0] - 1.0) < 1e-5


def test_smooth_scales_clamp_degenerate(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "tbr8_toy_layer.json")))
    a = np.array([0.0, 4.0, 0.0, 1e-7], np.float32)
    w = np.array([1.0, 0.0, 0.0, 1.0], np.float32)
    s = oracle.smooth_scales(a, w, 0.5)
    c = spec["clamp_min"]
    exp = [math.sqrt(c / 1.0), math.sqrt(4.0 / c), 1.0, math.sqrt(c / 1.0)]
    assert _rel(s, exp).max() < 1e-6
    assert np.all(np.isfinite(s)) and np.all(s > 0)


def test_static_scale_equals_brute_force():
    """ADR-010 point 1: max_j(act_max_j / s_j)/127 needs no calibration batches."""
    wl = synth.outlier_linear(M=8, K=256, N=64, calib_batches=5, calib_rows=33, x_dt=F16,
                              w_dt=F16, out_dt=F16, workload=91)
    am = np.zeros(wl.K, np.float32)
    for b in wl.calib:
        oracle.calib_absmax(b, F16, am)
    s = oracle.smooth_scales(am, oracle.calib_absmax(wl.w, F16), 0.5)
    a = oracle.static_scale(am, s)
    inv_s = np.array([oracle.recip(v) for v in s], np.float32)
    allx = np.concatenate([oracle.to_f32(b, F16) for b in wl.calib])
    smoothed = np.abs(allx * inv_s[None, :])                  # every calibration value, smoothed
    brute = np.float32(smoothed.max()) / np.float32(127.0)
    assert a == brute                                          # fl() is monotone: bit-exact


# --------------------------------------------------------------------------
# a4 weight quant, a5/a5' activation quant
# --------------------------------------------------------------------------

def _check_codes(v32, q, scale_rows, per_row=True):
    """Symmetric INT8 codes: in range, |v - q*scale| <= scale/2 (+ rounding), max -> +-127.

    per_row: every row's absmax element maps to +-127 (per-row scales);
    otherwise only the global absmax element does (one per-tensor scale).
    """
    assert q.min() >= -127 and q.max() <= 127
    v = v32.astype(np.float64)
    sc = np.asarray(scale_rows, np.float64)[:, None]
    err = np.abs(v - q.astype(np.float64) * sc)
    assert np.all(err <= sc * (0.5 + 1e-5) + 1e-30)
    if not per_row:
        assert np.abs(q.ravel()[np.argmax(np.abs(v))]) == 127
        return
    am = np.argmax(np.abs(v), axis=1)
    rows = np.arange(v.shape[0])
    nz = np.abs(v[rows, am]) > 0
    assert np.all(np.abs(q[rows, am])[nz] == 127)


@pytest.mark.parametrize("dt", [F32, F16, BF16])
def test_quant_weight_per_row(dt):
    g = np.random.default_rng(11)
    N, K = 37, 200
    W = synth.cast(g.standard_normal((N, K)).astype(np.float32) * 0.02, dt)
    s = (np.abs(g.standard_normal(K)) + 0.1).astype(np.float32)
    wq, ws = oracle.quant_weight(W, s, dt)
    Wp = oracle.to_f32(W, dt) * s[None, :]                    # W' = W diag(s): column j times s_j
    assert np.array_equal(ws, np.abs(Wp).max(axis=1) / np.float32(127))
    _check_codes(Wp, wq, ws)


def test_quant_weight_zero_row():
    W = np.zeros((2, 16), np.float32)
    W[1, 3] = -2.0
    wq, ws = oracle.quant_weight(W, np.ones(16, np.float32), F32)
    assert ws[0] == 0 and np.all(wq[0] == 0)
    assert wq[1, 3] == -127


@pytest.mark.parametrize("dt", [F32, F16, BF16])
def test_act_quant_static_and_per_token(dt):
    g = np.random.default_rng(12)
    M, K = 19, 136
    X = synth.cast(g.standard_normal((M, K)).astype(np.float32) * 4, dt)
    s = (np.abs(g.standard_normal(K)) + 0.2).astype(np.float32)
    inv = np.array([oracle.recip(v) for v in s], np.float32)
    Xs = oracle.to_f32(X, dt) * inv[None, :]                   # smoothing first (kwkr.cn 3.2)
    a = np.float32(np.abs(Xs).max() / np.float32(127))
    xq, av = oracle.smooth_quant_act(X, s, STATIC, a, dt)
    assert av[0] == a
    _check_codes(Xs, xq, np.full(M, a), per_row=False)
    # a static scale below the runtime max saturates rather than wraps
    xq_small, _ = oracle.smooth_quant_act(X, s, STATIC, a / 4, dt)
    assert xq_small.max() == 127 and xq_small.min() == -127
    xq2, a_tok = oracle.smooth_quant_act(X, s, PER_TOKEN, None, dt)
    assert np.array_equal(a_tok, np.abs(Xs).max(axis=1) / np.float32(127))
    _check_codes(Xs, xq2, a_tok)


# --------------------------------------------------------------------------
# a6 INT8 GEMM and dequant epilogue
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 16, 32), (7, 33, 48), (130, 65, 257), (3, 5, 1)])
def test_gemm_s32_vs_numpy(M, N, K):
    g = np.random.default_rng(M * 1000 + N)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (N, K), dtype=np.int8)
    acc = oracle.gemm_s32(A, B)
    assert np.array_equal(acc, A.astype(np.int64) @ B.astype(np.int64).T)


def test_gemm_s32_extreme_values():
    K = 4096
    A = np.full((2, K), -127, np.int8)
    B = np.full((3, K), 127, np.int8)
    B[1] = -127
    acc = oracle.gemm_s32(A, B)
    assert acc[0, 0] == -127 * 127 * K and acc[1, 1] == 127 * 127 * K


@pytest.mark.parametrize("out_dt", [F32, F16, BF16])
@pytest.mark.parametrize("mode", [STATIC, PER_TOKEN])
def test_dequant_vs_fp64(out_dt, mode):
    g = np.random.default_rng(5)
    M, N = 9, 40
    acc = g.integers(-2 ** 28, 2 ** 28, (M, N)).astype(np.int32)
    a = (np.abs(g.standard_normal(1 if mode == STATIC else M)) * 1e-3 + 1e-4).astype(np.float32)
    ws = (np.abs(g.standard_normal(N)) * 1e-4 + 1e-5).astype(np.float32)
    bias32 = g.standard_normal(N).astype(np.float32) * 100
    bias = synth.cast(bias32, out_dt)
    y = oracle.dequant(acc, a, mode, ws, out_dt, bias)
    yf = oracle.to_f32(y, out_dt).astype(np.float64)
    am = a.astype(np.float64)[0] if mode == STATIC else a.astype(np.float64)[:, None]
    ref = acc.astype(np.float64) * am * ws.astype(np.float64)[None, :] \
        + oracle.to_f32(bias, out_dt).astype(np.float64)[None, :]
    ulp_out = {F32: 2.0 ** -23, F16: 2.0 ** -10, BF16: 2.0 ** -7}[out_dt]
    mag = np.abs(acc.astype(np.float64) * am * ws.astype(np.float64)[None, :]) + np.abs(ref)
    # one rounding of (float)acc, one of a*w, one fma, one to the output type
    assert np.all(np.abs(yf - ref) <= mag * (3 * 2.0 ** -24) + np.abs(ref) * ulp_out + 1e-30)


def test_dequant_f32_hand_computed_roundings():
    """y = fl((float)acc * fl(a_m * w_n)), each rounding decided by hand:

    - acc = 2^24 + 1 widens to 2^24 (a tie, to even); times c = 3 that is
      50331648, where the exact product 50331651 would round to 50331652;
    - a = w = 1 + 2^-12: a*w = 1 + 2^-11 + 2^-24 rounds (a tie, to even) to
      c = 1 + 2^-11, and acc = 2^23 + 1 gives fl(8392705.000488...) = 8392705,
      where the unrounded a*w would give 8392706;
    - per-token rows use their own scale (a_1 = 1/4 halves row 1 against a_0 = 1/2)."""
    t = 1.0 + 2.0 ** -12
    acc = np.array([[2 ** 24 + 1, 2 ** 23 + 1, 3, -5],
                    [2 ** 24 + 1, 2 ** 23 + 1, 3, 0]], np.int64).astype(np.int32)
    # static: every row uses a[0]
    a_st = np.array([1.0], np.float32)
    ws = np.array([3.0, 1.0, 0.125, 0.5], np.float32)
    y = oracle.dequant_f32(acc, a_st, STATIC, ws)
    assert y[0, 0] == 50331648.0 and y[0, 2] == 0.375 and y[0, 3] == -2.5
    acc2 = np.array([[2 ** 23 + 1, 0]], np.int32)
    y2 = oracle.dequant_f32(acc2, np.array([t], np.float32), STATIC, np.array([t, 1.0], np.float32))
    assert y2[0, 0] == 8392705.0 and y2[0, 1] == 0.0
    # per token: row m uses a[m]
    a_pt = np.array([0.5, 0.25], np.float32)
    y3 = oracle.dequant_f32(acc, a_pt, PER_TOKEN, ws)
    assert y3[0, 2] == 3 * 0.0625 and y3[1, 2] == 3 * 0.03125
    assert y3[0, 0] == 2.0 ** 24 * 1.5 and y3[1, 0] == 2.0 ** 24 * 0.75
    assert y3[1, 3] == 0.0                         # no bias term: zero sums stay zero


@pytest.mark.parametrize("mode", [STATIC, PER_TOKEN])
def test_dequant_f32_bound_and_output_path(mode):
    """fp64 bound (one rounding each of (float)acc, a*w and the product) with a
    distinct scale per row, and equality with the rounded epilogue at fp32
    output without bias."""
    g = np.random.default_rng(15 + mode)
    M, N = 11, 37
    acc = g.integers(-2 ** 28, 2 ** 28, (M, N)).astype(np.int32)
    a = (np.abs(g.standard_normal(1 if mode == STATIC else M)) * 1e-3 + 1e-4).astype(np.float32)
    ws = (np.abs(g.standard_normal(N)) * 1e-4 + 1e-5).astype(np.float32)
    y = oracle.dequant_f32(acc, a, mode, ws)
    am = a.astype(np.float64)[0] if mode == STATIC else a.astype(np.float64)[:, None]
    ref = acc.astype(np.float64) * am * ws.astype(np.float64)[None, :]
    assert np.all(np.abs(y.astype(np.float64) - ref) <= np.abs(ref) * 3.01 * 2.0 ** -24)
    assert np.array_equal(y.view(np.uint32), oracle.dequant(acc, a, mode, ws, F32).view(np.uint32))


# --------------------------------------------------------------------------
# the identity, the quality claim and the ordering rule
# --------------------------------------------------------------------------

def _toy_state(outlier=True):
    wl = synth.linear_toy(outlier=outlier)
    return wl, oracle.calibrate_and_quantize(wl.calib, wl.w, 0.5)


def test_identity_fp64():
    """kwkr.cn 2.1: XW^T = (X diag(s)^-1)(W diag(s))^T, to 1e-9 relative in fp64."""
    wl, st = _toy_state()
    assert oracle.identity_residual(wl.x, wl.w, st.s) <= 1e-9
    s_wild = np.exp(np.random.default_rng(1).uniform(-6, 6, wl.K))
    assert oracle.identity_residual(wl.x, wl.w, s_wild) <= 1e-9


def test_identity_hand_computed_2x2():
    """The smoothed operands of a 2x2 case, worked by hand: s = (2, 1/2) halves
    column 0 of X and doubles column 0 of W (W is out x in: its columns are the
    input channels), and the product is unchanged."""
    X = np.array([[1.0, 2.0], [3.0, 4.0]])
    W = np.array([[5.0, 6.0], [7.0, 8.0]])
    Xs, Ws = oracle.smooth_operands(X, W, np.array([2.0, 0.5]))
    assert np.array_equal(Xs, [[0.5, 4.0], [1.5, 8.0]])
    assert np.array_equal(Ws, [[10.0, 3.0], [14.0, 4.0]])
    assert np.array_equal(Xs @ Ws.T, [[17.0, 23.0], [39.0, 53.0]])
    assert np.array_equal(X @ W.T, [[17.0, 23.0], [39.0, 53.0]])
    assert oracle.rel_residual(np.array([[3.0, 4.0]]), np.array([[3.0, 4.5]])) == 0.1


def test_identity_negative_controls():
    """The residual check is not vacuous: dividing X by s without scaling W (or
    scaling W alone) changes the product by far more than 1e-9 on the outlier
    layer, whose s spans two orders of magnitude."""
    wl, st = _toy_state()
    Y = wl.x.astype(np.float64) @ wl.w.astype(np.float64).T
    Xs, Ws = oracle.smooth_operands(wl.x, wl.w, st.s)
    assert oracle.rel_residual(Y, Xs @ wl.w.astype(np.float64).T) > 1e-2
    assert oracle.rel_residual(Y, wl.x.astype(np.float64) @ Ws.T) > 1e-2
    assert oracle.rel_residual(Y, Xs @ Ws.T) <= 1e-9


def _recon_err(wl, s, act_max):
    Y = wl.x.astype(np.float64) @ wl.w.astype(np.float64).T
    Yq = oracle.w8a8_output_f64(wl.x, wl.w, s, STATIC, act_max)
    return float(((Y - Yq) ** 2).sum())


def test_smoothing_gain_on_outlier_layer():
    """ADR-010 consequences: smoothing cuts the INT8 W+A output error on an outlier layer.

    The page reports about an order of magnitude for its own (unstated) test
    layer; on this toy law the factor is ~5.7 at alpha=0.5 and ~8.7 at the
    searched alpha.  The exact factor is not pinned; it is bounded below.
    """
    wl, st = _toy_state()
    plain = _recon_err(wl, np.ones(wl.K, np.float32), st.act_max)
    smooth = _recon_err(wl, st.s, st.act_max)
    assert plain / smooth >= 4.0
    best = max(plain / _recon_err(wl, oracle.smooth_scales(st.act_max, st.w_max, al), st.act_max)
               for al in oracle.ALPHA_GRID)
    assert best >= 8.0


def test_smoothing_not_worse_on_normal_activations():
    wl, st = _toy_state(outlier=False)
    plain = _recon_err(wl, np.ones(wl.K, np.float32), st.act_max)
    smooth = _recon_err(wl, st.s, st.act_max)
    assert plain / smooth >= 0.8


def test_scaling_after_quantisation_gives_no_gain():
    """kwkr.cn 5.2: multiplying by 1/s after the activations were quantised does not help."""
    wl, st = _toy_state()
    X = wl.x.astype(np.float32)
    Y = X.astype(np.float64) @ wl.w.astype(np.float64).T
    ones = np.ones(wl.K, np.float32)
    a_plain = oracle.static_scale(st.act_max, ones)
    xq, _ = oracle.smooth_quant_act(X, ones, STATIC, a_plain)           # quantise first ...
    x_deq = xq.astype(np.float64) * float(a_plain) / st.s.astype(np.float64)   # ... then scale
    wq, ws = oracle.quant_weight(wl.w, st.s)
    Yw = x_deq @ (wq.astype(np.float64) * ws.astype(np.float64)[:, None]).T
    wrong = float(((Y - Yw) ** 2).sum())
    plain = _recon_err(wl, ones, st.act_max)
    right = _recon_err(wl, st.s, st.act_max)
    assert wrong > 0.6 * plain and wrong > 3 * right


# --------------------------------------------------------------------------
# a7 alpha search
# --------------------------------------------------------------------------

def test_alpha_search_matches_fp64_reevaluation(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "adr010_defaults.json")))
    assert tuple(spec["alpha_grid"]) == oracle.ALPHA_GRID
    assert spec["alpha_default"] == oracle.ALPHA_DEFAULT
    wl = synth.heavy_13b(M=64, K=256, N=192, calib_batches=4, calib_rows=64)
    am = np.zeros(wl.K, np.float32)
    for b in wl.calib:
        oracle.calib_absmax(b, F16, am)
    wm = oracle.calib_absmax(wl.w, F16)
    held = wl.calib[0]
    best, mses, y_ref = oracle.alpha_search(held, wl.w, am, wm)
    # independent re-evaluation: numpy fp64 reference product and fp64 MSE
    Xh = synth.as_f16(held).astype(np.float64)
    Wf = synth.as_f16(wl.w).astype(np.float64)
    ref = (Xh @ Wf.T).astype(np.float16).astype(np.float64)
    assert np.max(np.abs(synth.as_f16(y_ref).astype(np.float64) - ref)) <= np.max(np.abs(ref)) * 2 ** -10
    again = []
    for al in oracle.ALPHA_GRID:
        s = oracle.smooth_scales(am, wm, al)
        a = oracle.static_scale(am, s)
        wq, ws = oracle.quant_weight(wl.w, s, F16)
        xq, _ = oracle.smooth_quant_act(held, s, STATIC, a, F16)
        y = (xq.astype(np.int64) @ wq.astype(np.int64).T).astype(np.float64) * float(a) * ws[None, :]
        y16 = y.astype(np.float16).astype(np.float64)
        again.append(float(np.mean((y16 - synth.as_f16(y_ref).astype(np.float64)) ** 2)))
    # the re-evaluation rounds the exact fp64 dequant product once to fp16 where
    # the oracle rounds fl((float)acc * fl(a * w_n)) (three fp32 roundings,
    # <= 3 * 2^-24 relative): the two fp16 outputs differ by one fp16 ulp
    # only where that fp32 error crosses an fp16 rounding boundary (a
    # ~3 * 2^-13 fraction of the elements), each changing d^2 by about
    # 2 |d| 2^-11 |y|, so the MSEs agree to ~1e-5 relative; 1e-4 (the
    # tolerance the alpha search is held to) bounds it
    assert _rel(mses, again).max() < 1e-4
    assert oracle.ALPHA_GRID[int(np.argmin(again))] == best
    assert mses[oracle.ALPHA_GRID.index(best)] <= min(mses[0], mses[-1])


def test_mse_f16_vs_numpy():
    g = np.random.default_rng(4)
    y = g.standard_normal(1000).astype(np.float16)
    r = g.standard_normal(1000).astype(np.float16)
    ref = float(np.mean((y.astype(np.float64) - r.astype(np.float64)) ** 2))
    assert abs(oracle.mse_f16(y.view(np.uint16), r.view(np.uint16)) - ref) <= 1e-12 * ref


# --------------------------------------------------------------------------
# a8 RMSNorm fold, a9 SiLU*mul
# --------------------------------------------------------------------------

def test_rmsnorm_fold_equals_unfused():
    """kwkr.cn 2.3/3.2: folding 1/s into the norm gain equals RMSNorm followed by x/s."""
    g = np.random.default_rng(21)
    M, d = 13, 320
    X = synth.cast(g.standard_normal((M, d)).astype(np.float32) * 2, BF16)
    gamma = g.uniform(0.5, 1.5, d).astype(np.float32)
    s = (np.abs(g.standard_normal(d)) + 0.3).astype(np.float32)
    eps = 1e-5
    x = oracle.to_f32(X, BF16).astype(np.float64)
    r = 1.0 / np.sqrt((x * x).mean(axis=1) + eps)
    y_unfused = (x * r[:, None]) * gamma[None, :] / s.astype(np.float64)[None, :]
    a = np.float32(np.abs(y_unfused).max() / 127)
    xq, rr = oracle.rmsnorm_quant(X, gamma, s, eps, a, BF16)
    assert _rel(rr, r).max() < 1e-6
    v = y_unfused / float(a)
    assert np.all(np.abs(xq - v) <= 0.5 + 1e-4)
    near_tie = np.abs(np.abs(v - np.floor(v)) - 0.5) < 1e-4
    assert np.array_equal(xq[~near_tie], np.clip(np.round(v), -127, 127)[~near_tie])
    # r_given overrides the computed r (used for staged parity)
    xq2, rr2 = oracle.rmsnorm_quant(X, gamma, s, eps, a, BF16, r_given=rr)
    assert np.array_equal(xq2, xq) and np.array_equal(rr2, rr)


def test_rmsnorm_absmax_vs_fp64():
    g = np.random.default_rng(22)
    M, d = 40, 256
    X = synth.cast(g.standard_normal((M, d)).astype(np.float32) * 3, BF16)
    gamma = g.uniform(0.5, 1.5, d).astype(np.float32)
    x = oracle.to_f32(X, BF16).astype(np.float64)
    r = 1.0 / np.sqrt((x * x).mean(axis=1) + 1e-5)
    ref = np.abs(x * r[:, None] * gamma[None, :]).max(axis=0)
    half = oracle.rmsnorm_absmax(X[:20], gamma, 1e-5, BF16)
    got = oracle.rmsnorm_absmax(X[20:], gamma, 1e-5, BF16, half)      # running max over two batches
    assert _rel(got, ref).max() < 3e-7


def test_silu_mul_closed_form():
    g = np.array([0.0, 1.0, -1.0, 20.0, -20.0, 3.5, -0.25], np.float32)
    u = np.array([5.0, 2.0, 2.0, 1.0, 1.0, -1.0, 4.0], np.float32)
    h = oracle.to_f32(oracle.silu_mul_bf16(g, u), BF16).astype(np.float64)
    ref = np.array([float(gi) / (1.0 + math.exp(-float(gi))) * float(ui) for gi, ui in zip(g, u)])
    assert h[0] == 0.0
    assert np.all(np.abs(h - ref) <= np.abs(ref) * 2 ** -8 + 1e-30)
    assert abs(h[3] - 20.0) <= 20 * 2 ** -8 and abs(h[4]) < 1e-6


def test_silu_mul_grid_through_exp_overflow():
    """silu on a dense grid out to |g| = 100, where exp(-g) overflows fp32
    (g < -88.7) and silu(g) * u falls below the smallest bf16 subnormal: the
    result follows the closed form within one bf16 rounding (2^-8 relative) or
    1e-30 absolute, is exactly 0 at g = 0, and tends to g * u for large g."""
    g = np.concatenate([np.linspace(-100, 100, 4001), [-88.0, 88.0, -89.0, 89.0, -100.0, 100.0]]).astype(np.float32)
    u = np.random.default_rng(3).uniform(-3, 3, g.size).astype(np.float32)
    h = oracle.to_f32(oracle.silu_mul_bf16(g, u), BF16).astype(np.float64)
    ref = np.array([float(gi) / (1.0 + math.exp(-float(gi))) * float(ui) for gi, ui in zip(g, u)])
    assert np.all(np.abs(h - ref) <= np.abs(ref) * 2 ** -8 + 1e-30)
    big = g >= 30
    assert np.all(np.abs(h[big] - g[big] * u[big].astype(np.float64)) <= np.abs(g[big] * u[big]) * 2 ** -8)
    assert np.all(np.abs(h[g <= -95]) < 1e-38)
    z = oracle.silu_mul_bf16(np.zeros(3, np.float32), np.array([1.0, -7.0, 1e30], np.float32))
    assert np.all(oracle.to_f32(z, BF16) == 0.0)


# --------------------------------------------------------------------------
# whole-layer sanity: the W8A8 output approximates the fp64 product
# --------------------------------------------------------------------------

def test_pipeline_output_close_to_fp64():
    wl = synth.outlier_linear(M=32, K=512, N=96, calib_batches=4, calib_rows=64, x_dt=F16,
                              w_dt=F16, out_dt=F32, workload=92)
    st = oracle.calibrate_and_quantize(wl.calib, wl.w, 0.5, F16, F16)
    _, _, _, y = oracle.linear_forward(st, wl.x, STATIC, F32, F16)
    Y = synth.as_f16(wl.x).astype(np.float64) @ synth.as_f16(wl.w).astype(np.float64).T
    rel = np.linalg.norm(y - Y) / np.linalg.norm(Y)
    assert rel < 0.05


# --------------------------------------------------------------------------
# FP8 (E4M3) variant ([AIU]: smoothing carries over to FP8)
# --------------------------------------------------------------------------

def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok].view(np.uint32), ref[ok].view(np.uint32))


def test_e4m3_encode_vs_torch_in_range():
    """Round to nearest, ties to even, on random values from the subnormals up
    to 448 and on every exact midpoint between neighbouring codes."""
    g = np.random.default_rng(50)
    v = (g.standard_normal(200000) * np.exp2(g.uniform(-12, 8.7, 200000))).astype(np.float32)
    v = v[np.abs(v) < 464]
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (pos[1:] + pos[:-1]) / 2)   # midpoints exact in fp32
    v = np.concatenate([v, mids, -mids, pos.astype(np.float32), np.float32([0.0, -0.0])])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_encode_saturates():
    """Beyond the largest finite value the conversion saturates (the reading
    taken for the quantiser; torch's cast gives NaN there)."""
    v = np.float32([464.0, 480.0, 1e6, -500.0, np.inf, -np.inf])
    assert list(oracle.e4m3_encode(v)) == [0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]
    assert oracle.e4m3_encode(np.float32([np.nan]))[0] == 0x7F


def test_fp8_quantisers_map_the_row_max_to_448():
    g = np.random.default_rng(51)
    X = synth.cast(g.standard_normal((37, 96)).astype(np.float32) * 3, BF16)
    s = (np.abs(g.standard_normal(96)) + 0.2).astype(np.float32)
    q, a = oracle.smooth_quant_act_fp8(X, s, PER_TOKEN, dt=BF16)
    dec = oracle.e4m3_decode(q).astype(np.float64)
    assert np.all(np.abs(dec).max(axis=1) == 448.0)
    xs = oracle.to_f32(X, BF16).astype(np.float64) / s.astype(np.float64)[None, :]
    v = xs / a.astype(np.float64)[:, None]
    # nearest E4M3: within half a spacing (2^-4 relative for normals, 2^-10 absolute below 2^-6)
    assert np.all(np.abs(dec - v) <= np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6))
    W = synth.cast(g.standard_normal((23, 96)).astype(np.float32) * 0.02, BF16)
    qw, sw = oracle.quant_weight_fp8(W, s, BF16)
    assert np.all(np.abs(oracle.e4m3_decode(qw)).max(axis=1) == 448.0)
    # static: a scale that puts the outlier beyond 448 saturates it
    qs, _ = oracle.smooth_quant_act_fp8(X, s, STATIC, a_scale=np.float32(a.min()), dt=BF16)
    assert np.abs(oracle.e4m3_decode(qs)).max() == 448.0


def test_static_scale_fp8_equals_brute_force():
    """The FP8 closed form max_j(act_max_j / s_j) / 448 equals the largest
    smoothed calibration value / 448 (fl() is monotone), bit for bit; the E4M3
    code of that value at this scale is 448 (0x7E)."""
    wl = synth.outlier_linear(M=16, K=256, N=64, calib_batches=3, calib_rows=32, x_dt=F16, w_dt=F16,
                              out_dt=F16, workload=93)
    am = np.zeros(wl.K, np.float32)
    for b in wl.calib:
        oracle.calib_absmax(b, F16, am)
    s = oracle.smooth_scales(am, oracle.calib_absmax(wl.w, F16), 0.5)
    a8 = oracle.static_scale_fp8(am, s)
    inv_s = np.where(s > 0, np.float32(1) / s, np.float32(0)).astype(np.float32)
    brute = max(float(np.abs((oracle.to_f32(b, F16) * inv_s[None, :]).astype(np.float32)).max()) for b in wl.calib)
    assert a8 == np.float32(np.float32(brute) / np.float32(448.0))
    assert np.float32(a8 * np.float32(448.0)) / np.float32(brute) == pytest.approx(1.0, abs=2 ** -22)
    q, _ = oracle.smooth_quant_act_fp8(np.concatenate(wl.calib), s, STATIC, a8, F16)
    assert (q & 0x7F).max() == 0x7E and oracle.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0


def test_gemm_fp8_f64_is_exact():
    """E4M3 values are multiples of 2^-9, so their products scaled by 2^18 are
    integers: the int64 matmul of the codes' values times 2^9 is the exact sum."""
    g = np.random.default_rng(52)
    xq = g.integers(0, 256, (9, 700), dtype=np.uint8)
    wq = g.integers(0, 256, (13, 700), dtype=np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0x7E                      # no NaN codes
    wq[(wq & 0x7F) == 0x7F] = 0xFE
    xi = np.rint(oracle.e4m3_decode(xq).astype(np.float64) * 512).astype(np.int64)
    wi = np.rint(oracle.e4m3_decode(wq).astype(np.float64) * 512).astype(np.int64)
    assert np.array_equal(xi.astype(np.float64) / 512, oracle.e4m3_decode(xq).astype(np.float64))
    exact = xi @ wi.T
    assert np.array_equal(oracle.gemm_fp8_f64(xq, wq) * 2.0 ** 18, exact.astype(np.float64))


# --------------------------------------------------------------------------
# follow-ups: cross-layer folding, fp16 scale storage ([ADR10])
# --------------------------------------------------------------------------

def test_fold_into_previous_identity():
    """Folding 1/s into the previous layer's output rows leaves the product of
    the two layers unchanged (fp64, up to the fp32 rounding of the folded
    weights), directly and through the gated MLP form h = silu(g) * u."""
    g = np.random.default_rng(60)
    Kp, K, N, M = 48, 64, 40, 9
    X = g.standard_normal((M, Kp)).astype(np.float32)
    Wp = (g.standard_normal((K, Kp)) * 0.1).astype(np.float32)
    Wg = (g.standard_normal((K, Kp)) * 0.1).astype(np.float32)
    W = (g.standard_normal((N, K)) * 0.1).astype(np.float32)
    s = (np.abs(g.standard_normal(K)) + 0.3).astype(np.float32)
    Wp2 = oracle.fold_into_previous(Wp, s).astype(np.float64)
    Ws = W.astype(np.float64) * s.astype(np.float64)[None, :]
    x = X.astype(np.float64)
    ref = (x @ Wp.astype(np.float64).T) @ W.astype(np.float64).T
    got = (x @ Wp2.T) @ Ws.T
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-6
    gate = x @ Wg.astype(np.float64).T
    silu = gate / (1.0 + np.exp(-gate))
    ref_h = (silu * (x @ Wp.astype(np.float64).T)) @ W.astype(np.float64).T
    got_h = (silu * (x @ Wp2.T)) @ Ws.T
    assert np.linalg.norm(got_h - ref_h) / np.linalg.norm(ref_h) < 1e-6


def test_scales_fp16_round_trip():
    g = np.random.default_rng(61)
    v = (np.abs(g.standard_normal(1000)) * np.exp2(g.uniform(-14, 10, 1000))).astype(np.float32)
    (got,) = oracle.scales_fp16(v)
    assert np.array_equal(got, v.astype(np.float16).astype(np.float32))

