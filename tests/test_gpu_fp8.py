"""FP8 (E4M3) variant on the GPU against the oracle (aiunderstanding.org,
"SmoothQuant 和激活量化": the smoothing carries over to FP8 tensor cores).

Quantisers: given the oracle's s (and static scale), the E4M3 codes and the
per-row / per-token scales are bit-exact.  GEMM (CTA pairs for M > 128, the
weight-streaming kernel with or without the cluster split below): the tensor cores sum the
exact E4M3 products in fp32 in an unspecified order, so y is compared with
the exact product (oracle.gemm_fp8_f64, fp64) within the fp32 summation
bound K * 2^-24 * sum_k |x_k w_k| times the dequant factor, plus the
epilogue's roundings.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import BF16, F16, F32, TORCH_DT, bits_equal, dev, host, mismatch_report, rand_x, rel_err

pytestmark = pytest.mark.gpu

sq = pytest.importorskip("w8a8_post_quantization_calib_b200")


def _sync():
    assert sq.sync_status() == 0


def _u8(n_or_shape):
    return torch.empty(n_or_shape, dtype=torch.uint8, device="cuda")


# ------------------------------------------------------------------ quantisers
@pytest.mark.parametrize("M,K,dt", [(300, 4096, F16), (7, 1000, BF16), (5, 11008, BF16), (1, 4096, F16),
                                    (64, 520, F32), (257, 8192, BF16)])
@pytest.mark.parametrize("mode", [oracle.STATIC, oracle.PER_TOKEN])
def test_act_quant_fp8(M, K, dt, mode):
    X = rand_x(M * 3 + K + mode, (M, K), dt, 2.0, outliers=max(1, K // 200))
    g = np.random.default_rng(K + M)
    s = (np.abs(g.standard_normal(K)) * 3 + 0.05).astype(np.float32)
    a = np.array([0.03], np.float32)
    xq = _u8((M, K))
    at = dev(a) if mode == oracle.STATIC else torch.empty(M, dtype=torch.float32, device="cuda")
    sq.smooth_quant_act_fp8(dev(X, dt), dev(s), mode, at, xq)
    _sync()
    q_r, a_r = oracle.smooth_quant_act_fp8(X, s, mode, a[0] if mode == oracle.STATIC else None, dt)
    got = host(xq)
    assert np.array_equal(got, q_r), mismatch_report(got, q_r)
    if mode == oracle.PER_TOKEN:
        assert bits_equal(host(at), a_r), mismatch_report(host(at), a_r)
    else:
        # the static scale is small enough that some values saturate at +-448
        assert ((got & 0x7F) == 0x7E).any()


@pytest.mark.parametrize("N,K,dt", [(384, 4096, F16), (33, 1000, BF16), (7, 11008, BF16), (128, 520, F32),
                                    (1024, 8192, BF16)])
def test_weight_quant_fp8(N, K, dt):
    W = rand_x(N + K, (N, K), dt, 0.02)
    W[0] = 0                                         # zero row: scale 0, codes 0
    g = np.random.default_rng(N * K)
    s = (np.abs(g.standard_normal(K)) * 3 + 0.05).astype(np.float32)
    wq = _u8((N, K))
    ws = torch.empty(N, dtype=torch.float32, device="cuda")
    sq.quant_weight_fp8(dev(W, dt), dev(s), wq, ws)
    _sync()
    q_r, s_r = oracle.quant_weight_fp8(W, s, dt)
    assert np.array_equal(host(wq), q_r), mismatch_report(host(wq), q_r)
    assert bits_equal(host(ws), s_r), mismatch_report(host(ws), s_r)
    assert host(ws)[0] == 0.0 and np.all(host(wq)[0] == 0)
    # each row's maximum maps to +-448 (code 0x7E)
    assert np.all((host(wq)[1:] & 0x7F).max(axis=1) == 0x7E)


@pytest.mark.parametrize("K", [4096, 28672])
def test_smooth_scales_fp8(K):
    g = np.random.default_rng(K)
    am = (np.abs(g.standard_normal(K)) * 2).astype(np.float32)
    am[g.choice(K, 20, replace=False)] *= 60
    wm = (np.abs(g.standard_normal(K)) * 0.05 + 1e-3).astype(np.float32)
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    a = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.smooth_scales_fp8(dev(am), dev(wm), 0.5, s, a)
    _sync()
    s_r = oracle.smooth_scales(am, wm, 0.5)
    assert rel_err(host(s), s_r).max() <= 1e-6
    # given the GPU's s, the closed-form E4M3 scale is exact
    assert host(a)[0] == oracle.static_scale_fp8(am, host(s))


# ------------------------------------------------------------------ GEMM
def _e4m3_codes(g, shape):
    """Random finite E4M3 codes (no 0x7F / 0xFF NaN codes)."""
    c = g.integers(0, 256, shape).astype(np.uint8)
    nan = (c & 0x7F) == 0x7F
    c[nan] ^= 0x01
    return c


def _check_fp8_gemm(xq, wq, a, mode, ws, bias32, out_dt, y):
    M, K = xq.shape
    N = wq.shape[0]
    acc = oracle.gemm_fp8_f64(xq, wq)                      # exact
    S = np.abs(oracle.e4m3_decode(xq).astype(np.float64)) @ np.abs(oracle.e4m3_decode(wq).astype(np.float64)).T
    am = a.astype(np.float64)[0] if mode == oracle.STATIC else a.astype(np.float64)[:, None]
    c = am * ws.astype(np.float64)[None, :]
    b = np.zeros(N) if bias32 is None else oracle.to_f32(synth.cast(bias32, out_dt), out_dt).astype(np.float64)
    ref = acc * c + b[None, :]
    got = oracle.to_f32(host(y), out_dt).astype(np.float64) if out_dt != F32 else host(y).astype(np.float64)
    ulp_out = {F32: 2.0 ** -23, F16: 2.0 ** -10, BF16: 2.0 ** -7}[out_dt]
    tol = np.abs(c) * S * K * 2.0 ** -24 + (np.abs(acc * c) + np.abs(ref)) * 3 * 2.0 ** -24 + np.abs(ref) * ulp_out \
        + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= tol), mismatch_report(got[err > tol], ref[err > tol])
    # the observed accumulation error, in units of the fp32 summation bound's unit
    return float((np.maximum(err - np.abs(ref) * ulp_out, 0) / np.maximum(np.abs(c) * S, 1e-300)).max())


@pytest.mark.parametrize("M,N,K", [(300, 528, 1040), (129, 256, 4096), (16, 1024, 2048), (1, 512, 1024),
                                   (512, 768, 11008), (1, 4096, 11008), (64, 1024, 4096), (128, 2048, 2048),
                                   (33, 11008, 4096), (100, 9600, 1040)])
@pytest.mark.parametrize("out_dt", [F32, F16, BF16])
def test_linear_fp8(M, N, K, out_dt):
    g = np.random.default_rng(M * 7 + N + K + out_dt)
    xq = _e4m3_codes(g, (M, K))
    wq = _e4m3_codes(g, (N, K))
    mode = oracle.PER_TOKEN if (M + N) % 2 else oracle.STATIC
    a = (np.abs(g.standard_normal(1 if mode == oracle.STATIC else M)) * 1e-2 + 1e-3).astype(np.float32)
    ws = (np.abs(g.standard_normal(N)) * 1e-3 + 1e-4).astype(np.float32)
    bias32 = (g.standard_normal(N) * 5).astype(np.float32) if out_dt != F32 else None
    y = torch.empty(M, N, dtype=TORCH_DT[out_dt], device="cuda")
    sq.linear_fp8(dev(xq), dev(wq), dev(a), mode, dev(ws), y,
                  bias=dev(synth.cast(bias32, out_dt), out_dt) if bias32 is not None else None)
    _sync()
    _check_fp8_gemm(xq, wq, a, mode, ws, bias32, out_dt, y)


def test_linear_fp8_exact_small_sums():
    """Codes whose products and partial sums are small integers: every fp32
    sum is exact, so y equals the oracle's fp64 product to the last bit."""
    g = np.random.default_rng(5)
    M, N, K = 256, 256, 512
    vals = np.array([0x00, 0x38, 0xB8, 0x40, 0xC0], np.uint8)      # 0, 1, -1, 2, -2
    xq = vals[g.integers(0, 5, (M, K))]
    wq = vals[g.integers(0, 5, (N, K))]
    a = np.array([1.0], np.float32)
    ws = np.ones(N, np.float32)
    y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    sq.linear_fp8(dev(xq), dev(wq), dev(a), oracle.STATIC, dev(ws), y)
    _sync()
    assert np.array_equal(host(y), oracle.gemm_fp8_f64(xq, wq).astype(np.float32))


# ------------------------------------------------------------------ the whole FP8 linear
def test_fp8_outlier_linear_pipeline():
    """Calibration -> smoothing -> FP8 weight / activation codes -> FP8 GEMM on
    the Llama-shaped outlier law: codes bit-exact with the oracle given the
    GPU's s and scale; the output within the GEMM bound of the exact product."""
    wl = synth.outlier_linear(M=256, K=2048, N=1024, calib_batches=4, calib_rows=256, x_dt=F16, w_dt=F16,
                              out_dt=F16, workload=71)
    act_max = torch.zeros(wl.K, dtype=torch.float32, device="cuda")
    for b in wl.calib:
        sq.calib_absmax(dev(b, F16), act_max)
    W = dev(wl.w, F16)
    w_max = torch.zeros(wl.K, dtype=torch.float32, device="cuda")
    sq.calib_absmax(W, w_max)
    s = torch.empty(wl.K, dtype=torch.float32, device="cuda")
    a = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.smooth_scales_fp8(act_max, w_max, 0.5, s, a)
    wq = _u8((wl.N, wl.K))
    ws = torch.empty(wl.N, dtype=torch.float32, device="cuda")
    sq.quant_weight_fp8(W, s, wq, ws)
    xq = _u8((wl.M, wl.K))
    sq.smooth_quant_act_fp8(dev(wl.x, F16), s, oracle.STATIC, a, xq)
    y = torch.empty(wl.M, wl.N, dtype=torch.float16, device="cuda")
    sq.linear_fp8(xq, wq, a, oracle.STATIC, ws, y)
    _sync()
    s_h, a_h = host(s), host(a)
    assert a_h[0] == oracle.static_scale_fp8(host(act_max), s_h)
    wq_r, ws_r = oracle.quant_weight_fp8(wl.w, s_h, F16)
    xq_r, _ = oracle.smooth_quant_act_fp8(wl.x, s_h, oracle.STATIC, a_h[0], F16)
    assert np.array_equal(host(wq), wq_r) and bits_equal(host(ws), ws_r)
    assert np.array_equal(host(xq), xq_r)
    _check_fp8_gemm(xq_r, wq_r, a_h, oracle.STATIC, ws_r, None, F16, y)
    # and the FP8 layer approximates the unquantised product
    Y = synth.as_f16(wl.x).astype(np.float64) @ synth.as_f16(wl.w).astype(np.float64).T
    yf = oracle.to_f32(host(y), F16).astype(np.float64)
    assert np.linalg.norm(yf - Y) / np.linalg.norm(Y) < 0.05      # the oracle gives 0.033 on this law
