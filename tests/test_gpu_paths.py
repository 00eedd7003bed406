"""Parity of the composed paths on the GPU (through the C ABI) against the oracle.

- the gate/up SiLU*mul epilogue at the edge values of g (0, +-20, +-88,
  +-100: exp(-g) overflowing fp32 and the fast division meeting a huge
  divisor) and with a zero requant scale;
- the alpha grid search, staged (the oracle's s, scale and reference product
  fed to the GPU's quantise -> GEMM -> squared-error chain) and whole;
- the column-parallel linear over 2 and 3 shards on the one GPU (pwwt.cn
  "SmoothQuant技术解析" 4.3: the statistic is combined across shards, every
  shard quantises and multiplies its own output rows, and the gathered
  columns equal the unsharded call bit for bit);
- the layer driver (Calibrator -> QuantizedLinear) against the oracle pipeline;
- whole chains on a created stream (programmatic dependent launches) equal
  to the same chains on the default stream (plain launches).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import BF16, F16, F32, bits_equal, dev, host, mismatch_report, rand_x, rel_err

pytestmark = pytest.mark.gpu

sq = pytest.importorskip("w8a8_post_quantization_calib_b200")


def _sync():
    assert sq.sync_status() == 0


def _gateup_order(Nh):
    return np.concatenate([np.concatenate([np.arange(b, b + 32), Nh + np.arange(b, b + 32)])
                           for b in range(0, Nh, 32)])


# ------------------------------------------------------------------ a9 edges
def test_gateup_silu_edge_values():
    """Rows 0..63 of A are one-hot at k = 0, so their gate sums are exactly
    Bg[c, 0] and their up sums Bu[c, 0]; with a = w_scale = 1 the gate values
    are g in {0, +-20, +-88, +-100} (and the up values small integers).  The
    other rows reach |g| ~ 1e5 (exp(-g) overflows fp32 for g < -88.7)."""
    M, Nh, K = 300, 128, 512
    g = np.random.default_rng(41)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    A[:64] = 0
    A[:64, 0] = 1
    Bg = g.integers(-127, 128, (Nh, K), dtype=np.int8)
    Bu = g.integers(-127, 128, (Nh, K), dtype=np.int8)
    edges = np.array([0, 20, -20, 88, -88, 100, -100, 89, -89, 87, -87, 1], np.int8)
    Bg[:, 0] = edges[np.arange(Nh) % len(edges)]
    Bu[:, 0] = np.array([1, -1, 3, -7, 127, -127], np.int8)[np.arange(Nh) % 6]
    a = np.array([1.0], np.float32)
    wsg = np.ones(Nh, np.float32)
    wsu = np.ones(Nh, np.float32)
    order = _gateup_order(Nh)
    Bgu = np.concatenate([Bg, Bu])[order]
    wsgu = np.concatenate([wsg, wsu])[order]
    s2 = (np.abs(g.standard_normal(Nh)) + 0.5).astype(np.float32)

    gv = oracle.dequant_f32(oracle.gemm_s32(A, Bg), a, oracle.STATIC, wsg)
    uv = oracle.dequant_f32(oracle.gemm_s32(A, Bu), a, oracle.STATIC, wsu)
    assert set(np.unique(gv[:64])) <= set(edges.astype(np.float32))
    h_ref = oracle.silu_mul_bf16(gv, uv)
    hf_ref = oracle.to_f32(h_ref, BF16).astype(np.float64)

    for a2v in (0.0, 1e3):
        a2 = np.array([a2v], np.float32)
        h = torch.empty(M, Nh, dtype=torch.bfloat16, device="cuda")
        hq = torch.full((M, Nh), 55, dtype=torch.int8, device="cuda")
        sq.linear_w8a8_gateup_silu(dev(A), dev(Bgu), dev(a), oracle.STATIC, dev(wsgu), h=h, s2=dev(s2),
                                   a2=dev(a2), hq=hq)
        _sync()
        h_got = host(h)
        hf_got = oracle.to_f32(h_got, BF16).astype(np.float64)
        assert np.all(np.isfinite(hf_got))
        # within 2 bf16 ulp of the correctly rounded SiLU, or 1e-30 absolute (the
        # fast division returns 0 for divisors in (2^126, 2^128), i.e. g near -88)
        ulp = np.maximum(np.abs(hf_ref), 1e-30) * 2.0 ** -7
        bad = np.abs(hf_got - hf_ref) > 2 * ulp + 1e-30
        assert not bad.any(), mismatch_report(hf_got[bad], hf_ref[bad])
        e = gv[:64] == 0
        assert np.all(hf_got[:64][e] == 0.0)                       # silu(0) * u = 0
        big = gv >= 20
        assert np.all(np.abs(hf_got[big] - gv[big] * uv[big]) <= np.abs(gv[big] * uv[big]) * 2.0 ** -6)
        assert np.all(np.abs(hf_got[gv <= -89]) < 1e-30)         # exp(-g) = inf: silu -> 0
        hq_got = host(hq)
        if a2v == 0.0:
            assert np.all(hq_got == 0)                              # zero scale: reciprocal 0, codes 0
        else:
            # staged: the requant of the GPU's own bf16 h is the oracle's, bit for bit
            hq_ref, _ = oracle.smooth_quant_act(h_got, s2, oracle.STATIC, a2[0], BF16)
            assert np.array_equal(hq_got, hq_ref), mismatch_report(hq_got, hq_ref)


# ------------------------------------------------------------------ a7
def _alpha_inputs(M_held, K, N, calib_batches):
    wl = synth.heavy_13b(M=64, K=K, N=N, calib_batches=calib_batches, calib_rows=M_held)
    am = np.zeros(wl.K, np.float32)
    for b in wl.calib:
        oracle.calib_absmax(b, F16, am)
    wm = oracle.calib_absmax(wl.w, F16)
    return wl, am, wm


@pytest.mark.parametrize("M_held,K,N", [(128, 512, 272), (512, 1024, 1536)])
def test_alpha_search_staged_chain(M_held, K, N):
    """Given the oracle's s, static scale and reference product, the GPU's
    per-alpha chain (weight quant, activation quant, INT8 GEMM with the fp16
    epilogue, fp64 squared-error sum) reproduces the oracle's MSE up to the
    order of the fp64 sum (1e-9 relative)."""
    wl, am, wm = _alpha_inputs(M_held, K, N, 4)
    held = wl.calib[0]
    best_r, mses_r, y_ref = oracle.alpha_search(held, wl.w, am, wm)
    W, X, Yr = dev(wl.w, F16), dev(held, F16), dev(y_ref, F16)
    for i, al in enumerate(oracle.ALPHA_GRID):
        s = oracle.smooth_scales(am, wm, al)
        a = np.array([oracle.static_scale(am, s)], np.float32)
        wq = torch.empty(N, K, dtype=torch.int8, device="cuda")
        ws = torch.empty(N, dtype=torch.float32, device="cuda")
        sq.quant_weight(W, dev(s), wq, ws)
        xq = torch.empty(M_held, K, dtype=torch.int8, device="cuda")
        sq.smooth_quant_act(X, dev(s), oracle.STATIC, dev(a), xq)
        y = torch.empty(M_held, N, dtype=torch.float16, device="cuda")
        sq.linear_w8a8(xq, wq, dev(a), oracle.STATIC, ws, y)
        sse = torch.zeros(1, dtype=torch.float64, device="cuda")
        sq.sse_f16(y, Yr, sse)
        _sync()
        mse = float(sse.item()) / (M_held * N)
        assert abs(mse - mses_r[i]) <= 1e-9 * mses_r[i], (al, mse, mses_r[i])


@pytest.mark.parametrize("M_held,K,N", [(128, 512, 272), (512, 1024, 1536)])
def test_alpha_search_whole(M_held, K, N):
    """sq_alpha_search with its own s and its tensor-core reference product
    (fp32 accumulation, one fp16 rounding) against the oracle's (fp64 sum):
    the same alpha, MSEs within 1e-4 relative.  Both differences move an fp16
    output or reference by one ulp on a small fraction of the elements, each
    changing d^2 by ~2|d| 2^-11 |y| with no common sign."""
    wl, am, wm = _alpha_inputs(M_held, K, N, 4)
    held = wl.calib[0]
    best_r, mses_r, _ = oracle.alpha_search(held, wl.w, am, wm)
    work = torch.zeros(sq.alpha_search_workspace_size(M_held, N, K, 4), dtype=torch.uint8, device="cuda")
    best, mses = sq.alpha_search(dev(held, F16), dev(wl.w, F16), dev(am), dev(wm), work)
    assert best == best_r
    assert rel_err(mses, mses_r).max() < 1e-4, (mses, mses_r)
    assert mses[list(oracle.ALPHA_GRID).index(best)] <= min(mses[0], mses[-1])


# ------------------------------------------------------------------ tensor-parallel column split
@pytest.mark.parametrize("world", [2, 3])
def test_column_parallel_shards_equal_unsharded(world):
    from w8a8_post_quantization_calib_b200.dist import column_shard
    M, K, N = 200, 1024, 1536
    wl = synth.outlier_linear(M=M, K=K, N=N, calib_batches=2, calib_rows=128, x_dt=F16, w_dt=F16,
                              out_dt=F16, workload=61)
    X = dev(wl.x, F16)
    W = dev(wl.w, F16)
    act_max = torch.zeros(K, dtype=torch.float32, device="cuda")
    for b in wl.calib:
        sq.calib_absmax(dev(b, F16), act_max)

    def linear_for(rows_w, w_max):
        s = torch.empty(K, dtype=torch.float32, device="cuda")
        a = torch.empty(1, dtype=torch.float32, device="cuda")
        sq.smooth_scales(act_max, w_max, 0.5, s, a)
        n = rows_w.shape[0]
        wq = torch.empty(n, K, dtype=torch.int8, device="cuda")
        ws = torch.empty(n, dtype=torch.float32, device="cuda")
        sq.quant_weight(rows_w, s, wq, ws)
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        sq.smooth_quant_act(X, s, oracle.STATIC, a, xq)
        y = torch.empty(M, n, dtype=torch.float16, device="cuda")
        sq.linear_w8a8(xq, wq, a, oracle.STATIC, ws, y)
        return y, s, a

    # unsharded
    w_max = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.calib_absmax(W, w_max)
    y_full, s_full, a_full = linear_for(W, w_max)
    # shards: each takes the weight column statistic over its own rows; the
    # all-reduce(MAX) across ranks is the elementwise max of the shards' vectors
    spans = [column_shard(N, r, world) for r in range(world)]
    parts = []
    for lo, hi in spans:
        m = torch.zeros(K, dtype=torch.float32, device="cuda")
        sq.calib_absmax(W[lo:hi], m)
        parts.append(m)
    w_max_sh = torch.stack(parts).amax(dim=0)
    outs = []
    for lo, hi in spans:
        y, s, a = linear_for(W[lo:hi].contiguous(), w_max_sh)
        assert torch.equal(s, s_full) and torch.equal(a, a_full)
        outs.append(y)
    _sync()
    y_sh = torch.cat(outs, dim=1)
    assert torch.equal(y_sh.view(torch.int16), y_full.view(torch.int16))
    # and the oracle on sampled rows (given the GPU's s and scale)
    s_h, a_h = host(s_full), host(a_full)
    wq_r, ws_r = oracle.quant_weight(wl.w, s_h, F16)
    rows = np.r_[0:8, M - 8:M]
    xq_r, a_r = oracle.smooth_quant_act(wl.x[rows], s_h, oracle.STATIC, a_h[0], F16)
    y_r = oracle.dequant(oracle.gemm_s32(xq_r, wq_r), a_r, oracle.STATIC, ws_r, F16)
    got = host(y_sh)[rows]
    assert np.array_equal(got, y_r), mismatch_report(got, y_r)


# ------------------------------------------------------------------ layer driver
@pytest.mark.parametrize("mode", [oracle.STATIC, oracle.PER_TOKEN])
def test_layer_driver_matches_oracle_pipeline(mode):
    from w8a8_post_quantization_calib_b200.layer import Calibrator, QuantizedLinear
    wl = synth.outlier_linear(M=96, K=512, N=384, calib_batches=3, calib_rows=64, x_dt=F16, w_dt=F16,
                              out_dt=F16, workload=62)
    cal = Calibrator(wl.K)
    for b in wl.calib:
        cal.add_batch(dev(b, F16))
    layer = QuantizedLinear.from_float(dev(wl.w, F16), cal.act_max, alpha=0.5, mode=mode)
    M = wl.x.shape[0]
    y = layer.forward(dev(wl.x, F16), out_dtype=torch.float16, workspace=layer.workspace(M))
    _sync()
    ref = oracle.calibrate_and_quantize(wl.calib, wl.w, 0.5, F16, F16)
    assert bits_equal(host(layer.act_max), ref.act_max)
    assert bits_equal(host(layer.w_max), ref.w_max)
    assert rel_err(host(layer.s), ref.s).max() <= 1e-6
    # the downstream steps are exact given the layer's own s and scale
    st = oracle.LinearState(ref.act_max, ref.w_max, host(layer.s), np.float32(host(layer.a_static)[0]),
                            *oracle.quant_weight(wl.w, host(layer.s), F16))
    assert bits_equal(host(layer.wq), st.wq) and bits_equal(host(layer.w_scale), st.w_scale)
    _, _, _, y_r = oracle.linear_forward(st, wl.x, mode, F16, F16)
    assert np.array_equal(host(y), y_r), mismatch_report(host(y), y_r)


# ------------------------------------------------------------------ created streams (programmatic launches)
def test_chains_on_a_created_stream_equal_the_default_stream():
    """On a created stream the kernels are launched with programmatic
    dependent launch (each one's prologue overlaps the previous kernel's
    tail); the results of whole chains must equal the default stream's bit
    for bit: the QKV-style linear (calibration -> scales -> weight codes ->
    activation codes -> GEMM), the robust quantile's four dependent
    passes, and the per-token small-M path."""
    wl = synth.outlier_linear(M=300, K=1024, N=768, calib_batches=3, calib_rows=256, x_dt=F16, w_dt=F16,
                              out_dt=F16, workload=63)
    calib = dev(np.concatenate(wl.calib), F16)
    W, X = dev(wl.w, F16), dev(wl.x, F16)

    def chain():
        am = torch.zeros(wl.K, dtype=torch.float32, device="cuda")
        sq.calib_absmax(calib, am)
        wm = torch.zeros(wl.K, dtype=torch.float32, device="cuda")
        sq.calib_absmax(W, wm)
        s = torch.empty(wl.K, dtype=torch.float32, device="cuda")
        a = torch.empty(1, dtype=torch.float32, device="cuda")
        sq.smooth_scales(am, wm, 0.5, s, a)
        wq = torch.empty(wl.N, wl.K, dtype=torch.int8, device="cuda")
        ws = torch.empty(wl.N, dtype=torch.float32, device="cuda")
        sq.quant_weight(W, s, wq, ws)
        outs = []
        for M, mode in ((300, oracle.STATIC), (16, oracle.PER_TOKEN)):
            xq = torch.empty(M, wl.K, dtype=torch.int8, device="cuda")
            at = a if mode == oracle.STATIC else torch.empty(M, dtype=torch.float32, device="cuda")
            sq.smooth_quant_act(X[:M], s, mode, at, xq)
            y = torch.empty(M, wl.N, dtype=torch.float16, device="cuda")
            sq.linear_w8a8(xq, wq, at, mode, ws, y)
            outs.append(y)
        q = torch.empty(wl.K, dtype=torch.float32, device="cuda")
        work = torch.empty(sq.calib_quantile_workspace_size(wl.K), dtype=torch.uint8, device="cuda")
        sq.calib_quantile(calib.float(), 0.999, q, work)       # fp32: four dependent digit passes
        return [am, wm, s, a, wq, ws, q] + outs

    ref = [t.clone() for t in chain()]
    _sync()
    side = torch.cuda.Stream()
    for _ in range(3):
        with torch.cuda.stream(side):
            got = chain()
        side.synchronize()
        _sync()
        for g, r in zip(got, ref):
            assert torch.equal(g.view(torch.uint8), r.view(torch.uint8))
    q_r = oracle.calib_quantile([oracle.to_f32(np.concatenate(wl.calib), F16)], 0.999, F32)
    assert bits_equal(host(ref[6]), q_r)


# ------------------------------------------------------------------ the h statistic in the gate/up epilogue
@pytest.mark.parametrize("M,Nh,K,mode", [(300, 256, 1024, oracle.STATIC), (1000, 384, 512, oracle.PER_TOKEN),
                                         (4096, 128, 2048, oracle.STATIC)])
def test_gateup_h_absmax_equals_the_statistic_of_h(M, Nh, K, mode):
    """sq_linear_w8a8_gateup_silu_absmax keeps the column max of |h| in the
    epilogue instead of writing h; it equals sq_calib_absmax over the h that
    sq_linear_w8a8_gateup_silu writes, bit for bit (both see the same
    bf16-rounded h), as a running max over two calls."""
    g = np.random.default_rng(M + Nh)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (2 * Nh, K), dtype=np.int8)
    a = (np.abs(g.standard_normal(1 if mode == oracle.STATIC else M)) * 2e-3 + 1e-4).astype(np.float32)
    ws = (np.abs(g.standard_normal(2 * Nh)) * 1e-3 + 1e-4).astype(np.float32)
    At, Bt, at, wst = dev(A), dev(B), dev(a), dev(ws)
    h = torch.empty(M, Nh, dtype=torch.bfloat16, device="cuda")
    sq.linear_w8a8_gateup_silu(At, Bt, at, mode, wst, h=h)
    ref = torch.zeros(Nh, dtype=torch.float32, device="cuda")
    sq.calib_absmax(h, ref)
    got = torch.zeros(Nh, dtype=torch.float32, device="cuda")
    sq.linear_w8a8_gateup_silu_absmax(At, Bt, at, mode, wst, got)
    _sync()
    assert torch.equal(got, ref)
    # a running max: a second batch (the first half of the rows) changes nothing, a scaled one raises it
    half = M // 2
    sq.linear_w8a8_gateup_silu_absmax(At[:half].contiguous(), Bt, at[:1] if mode == oracle.STATIC else at[:half],
                                      mode, wst, got)
    _sync()
    assert torch.equal(got, ref)
    # and against the oracle on the whole batch
    order = _gateup_order(Nh)
    inv = np.argsort(order)
    gv = oracle.dequant_f32(oracle.gemm_s32(A, B[inv][:Nh]), a, mode, ws[inv][:Nh])
    uv = oracle.dequant_f32(oracle.gemm_s32(A, B[inv][Nh:]), a, mode, ws[inv][Nh:])
    h_ref = np.abs(oracle.to_f32(oracle.silu_mul_bf16(gv, uv), BF16)).max(axis=0)
    assert np.all(np.abs(host(got) - h_ref) <= h_ref * 2.0 ** -6 + 1e-30)
