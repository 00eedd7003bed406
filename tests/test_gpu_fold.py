"""Cross-layer folding and fp16 scale storage on the GPU against the oracle
("010. SmoothQuant Integration": Alternative C -- fold 1/s into the previous
layer's weights -- and the consequences' fp16 storage of the scales).

Fold: the previous layer's weight rows are multiplied by fl(1/s_next) before
its own smoothing and per-row quantisation; given the same s and s_next the
codes and per-row scales are bit-exact with oracle.fold_into_previous followed
by oracle.quant_weight.  In the MLP block the fold goes into W_up's rows, and
the gate/up epilogue's requant then multiplies by recip(a2) only.

fp16 scales: the fp16 round trip equals the oracle's scales_fp16, and the GEMM
reading fp16 scales equals the GEMM given their exact fp32 widening.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import BF16, F16, F32, TORCH_DT, bits_equal, dev, host, mismatch_report, rand_x

pytestmark = pytest.mark.gpu

sq = pytest.importorskip("w8a8_post_quantization_calib_b200")


def _sync():
    assert sq.sync_status() == 0


def _gateup_order(Nh):
    return np.concatenate([np.concatenate([np.arange(b, b + 32), Nh + np.arange(b, b + 32)])
                           for b in range(0, Nh, 32)])


@pytest.mark.parametrize("N,K,dt", [(300, 4096, BF16), (7, 1000, F16), (257, 8192, BF16), (96, 520, F32)])
def test_fold_weight_matches_oracle(N, K, dt):
    W = rand_x(N + 3 * K, (N, K), dt, 0.02)
    g = np.random.default_rng(N * 11 + K)
    s = (np.abs(g.standard_normal(K)) * 3 + 0.05).astype(np.float32)
    s_next = np.exp(g.uniform(-3, 3, N)).astype(np.float32)
    wq = torch.empty(N, K, dtype=torch.int8, device="cuda")
    ws = torch.empty(N, dtype=torch.float32, device="cuda")
    sq.quant_weight_fold(dev(W, dt), dev(s), dev(s_next), wq, ws)
    _sync()
    Wf = oracle.fold_into_previous(oracle.to_f32(W, dt), s_next)
    wq_r, ws_r = oracle.quant_weight(Wf, s, F32)
    assert bits_equal(host(ws), ws_r), mismatch_report(host(ws), ws_r)
    assert np.array_equal(host(wq), wq_r), mismatch_report(host(wq), wq_r)


def test_gateup_fold_and_folded_requant():
    """MLP block (reduced): W_up's rows carry 1/s2; the gate/up GEMM with s2 =
    NULL requantises h' = silu(g) * u' with recip(a2) only.  Codes of the
    folded weights are bit-exact; h' is within 2 bf16 ulp of the oracle's
    silu(g) * u'; the requant of the GPU's own h' is bit-exact; and the folded
    block's codes agree with the unfolded block's (the same mathematics up to
    rounding) on all but a small fraction."""
    M, d, Nh = 300, 1024, 256
    g = np.random.default_rng(77)
    X = rand_x(5, (M, d), BF16, 1.0, outliers=5)
    Wg, Wu = rand_x(6, (Nh, d), BF16, 0.02), rand_x(7, (Nh, d), BF16, 0.02)
    s1 = (np.abs(g.standard_normal(d)) + 0.3).astype(np.float32)
    s2 = np.exp(g.uniform(-1.5, 1.5, Nh)).astype(np.float32)
    a1 = np.array([0.03], np.float32)
    a2 = np.array([0.004], np.float32)
    xq = torch.empty(M, d, dtype=torch.int8, device="cuda")
    sq.smooth_quant_act(dev(X, BF16), dev(s1), oracle.STATIC, dev(a1), xq)
    # folded and plain weights
    wq_f = torch.empty(2 * Nh, d, dtype=torch.int8, device="cuda")
    ws_f = torch.empty(2 * Nh, dtype=torch.float32, device="cuda")
    sq.quant_weight_gateup_fold(dev(Wg, BF16), dev(Wu, BF16), dev(s1), dev(s2), wq_f, ws_f)
    wq_p = torch.empty_like(wq_f)
    ws_p = torch.empty_like(ws_f)
    sq.quant_weight_gateup(dev(Wg, BF16), dev(Wu, BF16), dev(s1), wq_p, ws_p)
    h_f = torch.empty(M, Nh, dtype=torch.bfloat16, device="cuda")
    hq_f = torch.empty(M, Nh, dtype=torch.int8, device="cuda")
    sq.linear_w8a8_gateup_silu(xq, wq_f, dev(a1), oracle.STATIC, ws_f, h=h_f, a2=dev(a2), hq=hq_f)
    hq_p = torch.empty_like(hq_f)
    sq.linear_w8a8_gateup_silu(xq, wq_p, dev(a1), oracle.STATIC, ws_p, s2=dev(s2), a2=dev(a2), hq=hq_p)
    _sync()
    # folded weight codes: oracle fold of the up rows, then the shared-s transform
    order = _gateup_order(Nh)
    Wcat = np.concatenate([oracle.to_f32(Wg, BF16), oracle.fold_into_previous(oracle.to_f32(Wu, BF16), s2)])[order]
    wq_r, ws_r = oracle.quant_weight(Wcat, s1, F32)
    assert bits_equal(host(ws_f), ws_r) and np.array_equal(host(wq_f), wq_r)
    # h' against the oracle's SiLU on the folded weights
    inv = np.argsort(order)
    xq_h = host(xq)
    gv = oracle.dequant_f32(oracle.gemm_s32(xq_h, wq_r[inv][:Nh]), a1, oracle.STATIC, ws_r[inv][:Nh])
    uv = oracle.dequant_f32(oracle.gemm_s32(xq_h, wq_r[inv][Nh:]), a1, oracle.STATIC, ws_r[inv][Nh:])
    h_ref = oracle.to_f32(oracle.silu_mul_bf16(gv, uv), BF16).astype(np.float64)
    h_got = host(h_f)
    hf = oracle.to_f32(h_got, BF16).astype(np.float64)
    assert np.all(np.abs(hf - h_ref) <= 2 * np.abs(h_ref) * 2.0 ** -7 + 1e-30)
    # the folded requant: q(fl(h' * recip(a2))), i.e. sq_smooth_quant_act with s = 1
    hq_r, _ = oracle.smooth_quant_act(h_got, np.ones(Nh, np.float32), oracle.STATIC, a2[0], BF16)
    assert np.array_equal(host(hq_f), hq_r), mismatch_report(host(hq_f), hq_r)
    # folded vs unfolded block: the same mathematics, rounded differently (the
    # fold rounds W_up * recip(s2) to fp32 before the transform, the per-row
    # scales change, and h' is rounded to bf16 -- 2^-9 relative -- where the
    # unfolded path rounds h and then multiplies by recip(s2)).  A bf16
    # rounding moves a code of magnitude v by up to v * 2^-8 / 2, so codes
    # near 127 flip at a rate of ~25 % and small codes rarely: every code
    # within 1, and a minority of them different.
    diff = np.abs(host(hq_f).astype(int) - host(hq_p).astype(int))
    assert diff.max() <= 1 and (diff != 0).mean() < 0.10


@pytest.mark.parametrize("n", [1, 1000, 65537])
def test_scales_f16_round_trip(n):
    g = np.random.default_rng(n)
    v = np.exp(g.uniform(-30, 12, n)).astype(np.float32)          # fp16 subnormals to overflow
    v[: min(n, 4)] = np.array([0.0, 6.1e-5, 65504.0, 70000.0], np.float32)[: min(n, 4)]
    h = torch.empty(n, dtype=torch.float16, device="cuda")
    sq.scales_to_f16(dev(v), h)
    back = torch.empty(n, dtype=torch.float32, device="cuda")
    sq.scales_from_f16(h, back)
    _sync()
    (want,) = oracle.scales_fp16(v)
    assert bits_equal(host(back), want), mismatch_report(host(back), want)


@pytest.mark.parametrize("M,N,K,mode", [(300, 528, 1040, oracle.STATIC), (16, 1024, 2048, oracle.PER_TOKEN),
                                        (1, 4096, 4096, oracle.PER_TOKEN), (512, 768, 4096, oracle.PER_TOKEN),
                                        (100, 11008, 4096, oracle.PER_TOKEN)])
@pytest.mark.parametrize("out_dt", [F16, BF16])
def test_linear_f16_scales(M, N, K, mode, out_dt):
    g = np.random.default_rng(M + N + K)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (N, K), dtype=np.int8)
    a32 = (np.abs(g.standard_normal(1 if mode == oracle.STATIC else M)) * 1e-2 + 1e-3).astype(np.float32)
    w32 = (np.abs(g.standard_normal(N)) * 1e-4 + 1e-5).astype(np.float32)
    a16, w16 = synth.cast(a32, F16), synth.cast(w32, F16)        # fp16 storage (bits)
    a_w, w_w = oracle.scales_fp16(a32, w32)                       # the widened values
    y16 = torch.empty(M, N, dtype=TORCH_DT[out_dt], device="cuda")
    work = torch.zeros(max(16, sq.linear_workspace_size(M, N, K)), dtype=torch.uint8, device="cuda")
    sq.linear_w8a8_f16scales(dev(A), dev(B), dev(a16, F16), mode, dev(w16, F16), y16, workspace=work)
    y32 = torch.empty_like(y16)
    sq.linear_w8a8(dev(A), dev(B), dev(a_w), mode, dev(w_w), y32, workspace=work)
    _sync()
    assert torch.equal(y16.view(torch.int16), y32.view(torch.int16))
    rows = np.r_[0:min(M, 8), max(0, M - 8):M]
    acc = oracle.gemm_s32(A[rows], B)
    y_r = oracle.dequant(acc, a_w if mode == oracle.STATIC else a_w[rows], mode, w_w, out_dt)
    assert np.array_equal(host(y16)[rows], y_r)
