"""Kernel-by-kernel parity of the CUDA path (through the C ABI) against the CPU oracle.

Both sides get the same seeded inputs; where a step consumes scales, the
oracle's scales are uploaded to the GPU, so codes and accumulators are
compared bit for bit ("given identical fp32 scales, INT8 tensors and INT32
accumulators are bit-exact").  Shapes span several tiles and ragged tails.
"""
import functools

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


@functools.lru_cache(maxsize=16)
def _int8_operands(M, N, K, seed):
    g = np.random.default_rng(seed)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (N, K), dtype=np.int8)
    return A, B, oracle.gemm_s32(A, B)


# ------------------------------------------------------------------ a1/a2
@pytest.mark.parametrize("dt", [F32, F16, BF16])
@pytest.mark.parametrize("rows,cols", [(1, 64), (37, 200), (1000, 4096), (3, 11008), (2049, 520)])
def test_calib_absmax(dt, rows, cols):
    b1 = rand_x(rows * 7 + cols, (rows, cols), dt, 3.0, outliers=min(5, cols // 8))
    b2 = rand_x(rows * 7 + cols + 1, (max(1, rows // 2), cols), dt, 3.0)
    am = torch.zeros(cols, dtype=torch.float32, device="cuda")
    sq.calib_absmax(dev(b1, dt), am)
    sq.calib_absmax(dev(b2, dt), am)
    _sync()
    ref = np.zeros(cols, np.float32)
    oracle.calib_absmax(b1, dt, ref)
    oracle.calib_absmax(b2, dt, ref)
    got = host(am)
    assert bits_equal(got, ref), mismatch_report(got, ref)


def test_calib_absmax_strided_rows():
    x = rand_x(5, (64, 96), F16, 2.0)            # view of the first 80 columns, ld = 96
    am = torch.zeros(80, dtype=torch.float32, device="cuda")
    t = dev(x, F16)
    sq.calib_absmax(t[:, :80], am)
    _sync()
    ref = np.abs(oracle.to_f32(x, F16)[:, :80]).max(axis=0)
    assert bits_equal(host(am), ref)


def test_calib_absmax_empty_is_noop():
    am = torch.full((16,), 3.0, dtype=torch.float32, device="cuda")
    x = torch.zeros(0, 16, dtype=torch.float16, device="cuda")
    sq.lib().sq_calib_absmax(x.data_ptr() or 16, 1, 0, 16, 16, am.data_ptr(), None)
    _sync()
    assert torch.all(am == 3.0)


# ------------------------------------------------------------------ a3
@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.75, 1.0, 0.6])
@pytest.mark.parametrize("K", [1, 1000, 28672])
def test_smooth_scales(alpha, K):
    g = np.random.default_rng(K)
    a = (np.abs(g.standard_normal(K)) * 5).astype(np.float32)
    w = (np.abs(g.standard_normal(K)) * 0.05).astype(np.float32)
    a[::97] = 0.0
    w[::89] = 0.0
    a[::13] *= 80
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    at = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.smooth_scales(dev(a), dev(w), alpha, s, at)
    _sync()
    s_ref = oracle.smooth_scales(a, w, alpha)
    a_ref = oracle.static_scale(a, s_ref)
    got = host(s)
    assert rel_err(got, s_ref).max() <= 1e-6
    assert (got != s_ref).mean() < 1e-3            # fp64 pow on both sides: rounding ties only
    assert rel_err(host(at), [a_ref]).max() <= 1e-6


# ------------------------------------------------------------------ a4
@pytest.mark.parametrize("dt", [F32, F16, BF16])
@pytest.mark.parametrize("N,K", [(300, 4096), (64, 5120), (3, 40), (17, 28672), (130, 1000), (300, 28672),
                                 (150, 20000)])
def test_quant_weight(dt, N, K):
    W = rand_x(N + K, (N, K), dt, 0.02)
    s = (np.abs(np.random.default_rng(K).standard_normal(K)) + 0.05).astype(np.float32)
    wq = torch.empty(N, K, dtype=torch.int8, device="cuda")
    ws = torch.empty(N, dtype=torch.float32, device="cuda")
    sq.quant_weight(dev(W, dt), dev(s), wq, ws)
    _sync()
    wq_ref, ws_ref = oracle.quant_weight(W, s, dt)
    assert bits_equal(host(ws), ws_ref), mismatch_report(host(ws), ws_ref)
    assert bits_equal(host(wq), wq_ref), mismatch_report(host(wq), wq_ref)


def test_quant_weight_zero_rows():
    W = np.zeros((40, 64), np.float32)
    W[7, 3] = 1.5
    s = np.ones(64, np.float32)
    wq = torch.empty(40, 64, dtype=torch.int8, device="cuda")
    ws = torch.empty(40, dtype=torch.float32, device="cuda")
    sq.quant_weight(dev(W), dev(s), wq, ws)
    _sync()
    wq_ref, ws_ref = oracle.quant_weight(W, s, F32)
    assert bits_equal(host(wq), wq_ref) and bits_equal(host(ws), ws_ref)


@pytest.mark.parametrize("dt", [F16, BF16])
def test_quant_weight_gateup_interleave(dt):
    Nh, K = 96, 512
    Wg = rand_x(1, (Nh, K), dt, 0.02)
    Wu = rand_x(2, (Nh, K), dt, 0.02)
    s = (np.abs(np.random.default_rng(3).standard_normal(K)) + 0.1).astype(np.float32)
    wq = torch.empty(2 * Nh, K, dtype=torch.int8, device="cuda")
    ws = torch.empty(2 * Nh, dtype=torch.float32, device="cuda")
    sq.quant_weight_gateup(dev(Wg, dt), dev(Wu, dt), dev(s), wq, ws)
    _sync()
    # interleaved order: blocks of 64 rows = 32 gate rows then the same 32 up rows
    order = np.concatenate([np.concatenate([np.arange(b, b + 32), Nh + np.arange(b, b + 32)])
                            for b in range(0, Nh, 32)])
    Wcat = np.concatenate([Wg, Wu])[order]
    wq_ref, ws_ref = oracle.quant_weight(Wcat, s, dt)
    assert bits_equal(host(wq), wq_ref) and bits_equal(host(ws), ws_ref)


# ------------------------------------------------------------------ a5 / a5'
@pytest.mark.parametrize("dt", [F32, F16, BF16])
@pytest.mark.parametrize("M,K", [(1, 4096), (300, 4096), (7, 11008), (5, 1024), (3, 40), (129, 5120),
                                 (200, 20000)])
@pytest.mark.parametrize("mode", [oracle.STATIC, oracle.PER_TOKEN])
def test_smooth_quant_act(dt, M, K, mode):
    X = rand_x(M * 3 + K, (M, K), dt, 2.0, outliers=min(8, K // 10))
    s = (np.abs(np.random.default_rng(K + 1).standard_normal(K)) + 0.2).astype(np.float32)
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    if mode == oracle.STATIC:
        a = np.float32(30.0 / 127)                 # saturates the outlier columns on purpose
        at = dev(np.array([a], np.float32))
        sq.smooth_quant_act(dev(X, dt), dev(s), mode, at, xq)
        _sync()
        xq_ref, _ = oracle.smooth_quant_act(X, s, oracle.STATIC, a, dt)
    else:
        at = torch.empty(M, dtype=torch.float32, device="cuda")
        sq.smooth_quant_act(dev(X, dt), dev(s), mode, at, xq)
        _sync()
        xq_ref, a_ref = oracle.smooth_quant_act(X, s, oracle.PER_TOKEN, None, dt)
        assert bits_equal(host(at), a_ref), mismatch_report(host(at), a_ref)
    assert bits_equal(host(xq), xq_ref), mismatch_report(host(xq), xq_ref)


@pytest.mark.parametrize("M", [1, 3, 100, 147])
@pytest.mark.parametrize("K,dt", [(2048, BF16), (4096, F16), (8192, BF16), (11008, BF16), (2048, F32)])
def test_row_split_kernels(M, K, dt):
    """Fewer rows than SMs take the cluster-split kernel (2, 4 or 8 CTAs per
    row, row reductions through distributed shared memory): per-token
    activation quant, weight transform and RMSNorm + quant, bit for bit."""
    X = rand_x(M * 7 + K, (M, K), dt, 1.5, outliers=min(8, K // 100))
    g = np.random.default_rng(M + K)
    s = (np.abs(g.standard_normal(K)) + 0.3).astype(np.float32)
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    at = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.smooth_quant_act(dev(X, dt), dev(s), oracle.PER_TOKEN, at, xq)
    _sync()
    xq_ref, a_ref = oracle.smooth_quant_act(X, s, oracle.PER_TOKEN, None, dt)
    assert bits_equal(host(at), a_ref), mismatch_report(host(at), a_ref)
    assert bits_equal(host(xq), xq_ref), mismatch_report(host(xq), xq_ref)
    ws = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.quant_weight(dev(X, dt), dev(s), xq, ws)
    _sync()
    wq_ref, ws_ref = oracle.quant_weight(X, s, dt)
    assert bits_equal(host(ws), ws_ref), mismatch_report(host(ws), ws_ref)
    assert bits_equal(host(xq), wq_ref), mismatch_report(host(xq), wq_ref)
    if dt != F32:
        gamma = g.uniform(0.5, 1.5, K).astype(np.float32)
        a = np.float32(0.04)
        r = torch.empty(M, dtype=torch.float32, device="cuda")
        sq.rmsnorm_quant(dev(X, dt), dev(gamma), dev(s), 1e-5, dev(np.array([a])), xq, r)
        _sync()
        xq_ref, r_ref = oracle.rmsnorm_quant(X, gamma, s, 1e-5, a, dt)
        assert bits_equal(host(r), r_ref), mismatch_report(host(r), r_ref)
        assert bits_equal(host(xq), xq_ref), mismatch_report(host(xq), xq_ref)
        am = torch.zeros(K, dtype=torch.float32, device="cuda")
        sq.rmsnorm_absmax(dev(X, dt), dev(gamma), 1e-5, am)
        _sync()
        am_ref = oracle.rmsnorm_absmax(X, gamma, 1e-5, dt)
        assert bits_equal(host(am), am_ref), mismatch_report(host(am), am_ref)


@pytest.mark.parametrize("M,K,dt", [(1, 16, F16), (37, 4104, BF16), (2049, 520, F32), (600, 4096, F16)])
def test_quant_static_streaming_misaligned_s(M, K, dt):
    """Static-scale quantisation (column strips x row slabs) with a 1/s vector
    that is not 16-byte aligned (scalar constant path) and ragged slabs."""
    X = rand_x(M + K * 5, (M, K), dt, 2.0, outliers=min(8, K // 10))
    s = (np.abs(np.random.default_rng(K).standard_normal(K)) + 0.2).astype(np.float32)
    s_buf = torch.zeros(K + 1, dtype=torch.float32, device="cuda")
    s_buf[1:] = dev(s)
    s_view = s_buf[1:]                              # 4-byte offset
    a = np.float32(20.0 / 127)
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sq.smooth_quant_act(dev(X, dt), s_view, oracle.STATIC, dev(np.array([a], np.float32)), xq)
    _sync()
    xq_ref, _ = oracle.smooth_quant_act(X, s, oracle.STATIC, a, dt)
    assert bits_equal(host(xq), xq_ref), mismatch_report(host(xq), xq_ref)


# ------------------------------------------------------------------ a8
@pytest.mark.parametrize("M,d", [(300, 8192), (5, 1000), (1, 4096)])
@pytest.mark.parametrize("random_gamma", [False, True])
def test_rmsnorm_quant(M, d, random_gamma):
    X = rand_x(M + d, (M, d), BF16, 1.0, outliers=max(1, d // 200))
    g = np.random.default_rng(d)
    gamma = g.uniform(0.5, 1.5, d).astype(np.float32) if random_gamma else np.ones(d, np.float32)
    s = (np.abs(g.standard_normal(d)) + 0.3).astype(np.float32)
    a = np.float32(0.05)
    xq = torch.empty(M, d, dtype=torch.int8, device="cuda")
    r = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.rmsnorm_quant(dev(X, BF16), dev(gamma), dev(s), 1e-5, dev(np.array([a])), xq, r)
    _sync()
    xq_ref, r_ref = oracle.rmsnorm_quant(X, gamma, s, 1e-5, a, BF16)
    assert bits_equal(host(r), r_ref), mismatch_report(host(r), r_ref)
    assert bits_equal(host(xq), xq_ref), mismatch_report(host(xq), xq_ref)


@pytest.mark.parametrize("sign", [1, -1, 0])
def test_rmsnorm_quant_saturation_boundary(sign):
    """Codes at the edge of saturation.  The kernel skips the clamp for the
    values of a thread whose magnitudes all lie below 127.5; a value of
    magnitude >= 127.5 rounds to +-128 and must be clamped to +-127.  The
    static scale is swept ulp by ulp so that row 0's largest value v =
    fl(y * fl(1/a)) falls on both sides of 127.5 (and on it where the
    rounding allows); the outlier of row 0 is positive, negative, or one of
    each.  Every row is compared with the oracle at every scale (300 rows:
    the many-row kernel; fewer rows than SMs take the split-row kernel)."""
    M, d = 300, 4096
    X = rand_x(40 + sign, (M, d), BF16, 1.0)
    xf = oracle.to_f32(X, BF16).copy()
    if sign >= 0:
        xf[0, 100] = 12.0
    if sign <= 0:
        xf[0, 2000] = -12.0
    X = synth.cast(xf, BF16)
    g = np.random.default_rng(41)
    gamma = g.uniform(0.5, 1.5, d).astype(np.float32)
    s = (np.abs(g.standard_normal(d)) + 0.3).astype(np.float32)
    s[[100, 2000]] = 1.0
    gamma[[100, 2000]] = 1.0
    # y of row 0 as the oracle computes it: fl(fl(x * r) * fl(gamma * fl(1/s)))
    _, r0 = oracle.rmsnorm_quant(X[:1], gamma, s, 1e-5, np.float32(1.0), BF16)
    c = (gamma * (np.float32(1.0) / s)).astype(np.float32)
    y0 = ((oracle.to_f32(X[:1], BF16) * r0[0]).astype(np.float32) * c).astype(np.float32)
    a0 = np.float32(np.abs(y0).max() / np.float32(127.5))
    vs = []
    for k in range(-6, 7):
        a = np.float32(a0)
        for _ in range(abs(k)):
            a = np.nextafter(a, np.float32(np.inf if k > 0 else 0), dtype=np.float32)
        vs.append(float(np.abs(y0 * (np.float32(1.0) / a)).max()))
        xq = torch.empty(M, d, dtype=torch.int8, device="cuda")
        sq.rmsnorm_quant(dev(X, BF16), dev(gamma), dev(s), 1e-5, dev(np.array([a], np.float32)), xq)
        _sync()
        xq_ref, _ = oracle.rmsnorm_quant(X, gamma, s, 1e-5, a, BF16)
        assert bits_equal(host(xq), xq_ref), (k, mismatch_report(host(xq), xq_ref))
        assert np.abs(xq_ref[0]).max() == 127
    assert min(vs) < 127.5 <= max(vs)


@pytest.mark.parametrize("dt", [BF16, F16])
def test_quant_static_saturation_boundary(dt):
    """Static-scale activation codes at the edge of saturation: the kernel
    clamps only the vectors holding a value of magnitude >= 127.5.  Rows 0-2
    carry +12, -12 and both; with s = 1 the scale is swept ulp by ulp around
    12 / 127.5, so that fl(12 * fl(1/a)) falls on both sides of 127.5."""
    M, K = 600, 4096
    xf = oracle.to_f32(rand_x(50, (M, K), dt, 1.0), dt).copy()
    xf[0, 8] = 12.0
    xf[1, 4000] = -12.0
    xf[2, 17], xf[2, 18] = 12.0, -12.0
    X = synth.cast(xf, dt)
    s = np.ones(K, np.float32)
    a0 = np.float32(np.float32(12.0) / np.float32(127.5))
    vs = []
    for k in range(-6, 7):
        a = np.float32(a0)
        for _ in range(abs(k)):
            a = np.nextafter(a, np.float32(np.inf if k > 0 else 0), dtype=np.float32)
        vs.append(float(np.float32(12.0) * (np.float32(1.0) / a)))
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        sq.smooth_quant_act(dev(X, dt), dev(s), oracle.STATIC, dev(np.array([a], np.float32)), xq)
        _sync()
        xq_ref, _ = oracle.smooth_quant_act(X, s, oracle.STATIC, a, dt)
        assert bits_equal(host(xq), xq_ref), (k, mismatch_report(host(xq), xq_ref))
    assert min(vs) < 127.5 <= max(vs)


# ------------------------------------------------------------------ a6
GEMM_SHAPES = [(1, 16, 32), (16, 48, 48), (100, 272, 1040), (128, 528, 4096), (129, 256, 128),
               (300, 528, 1040), (64, 4096, 11008), (257, 768, 4096)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_s32(M, N, K):
    g = np.random.default_rng(M * 131 + N * 7 + K)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (N, K), dtype=np.int8)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    sq.gemm_s32(dev(A), dev(B), acc)
    _sync()
    ref = oracle.gemm_s32(A, B)
    got = host(acc)
    assert np.array_equal(got, ref), mismatch_report(got, ref)


def test_gemm_s32_extremes():
    K = 8192
    A = np.full((130, K), -127, np.int8)
    B = np.full((32, K), 127, np.int8)
    B[1::2] = -127
    acc = torch.empty(130, 32, dtype=torch.int32, device="cuda")
    sq.gemm_s32(dev(A), dev(B), acc)
    _sync()
    assert np.array_equal(host(acc), oracle.gemm_s32(A, B))


@pytest.mark.parametrize("M,N,K", [(1, 16, 32), (5, 272, 1040), (16, 4096, 11008), (64, 528, 4096),
                                   (128, 256, 256), (200, 528, 1040), (300, 4096, 512)])
@pytest.mark.parametrize("out_dt", [F32, F16, BF16])
@pytest.mark.parametrize("mode", [oracle.STATIC, oracle.PER_TOKEN])
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("with_ws", [False, True])
def test_linear_w8a8(M, N, K, out_dt, mode, with_bias, with_ws):
    if with_ws and M > 128:
        pytest.skip("workspace only used by the small-M path")
    A, B, acc_ref = _int8_operands(M, N, K, M * 7 + N * 3 + K)
    g = np.random.default_rng(M + N + K + out_dt)
    a = (np.abs(g.standard_normal(1 if mode == oracle.STATIC else M)) * 1e-2 + 1e-3).astype(np.float32)
    ws = (np.abs(g.standard_normal(N)) * 1e-4 + 1e-5).astype(np.float32)
    bias = synth.cast(g.standard_normal(N).astype(np.float32), out_dt) if with_bias else None
    y = torch.empty(M, N, dtype={F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}[out_dt],
                    device="cuda")
    work = None
    if with_ws:
        n = sq.linear_workspace_size(M, N, K)
        work = torch.zeros(n, dtype=torch.uint8, device="cuda")
    for _ in range(2):      # twice: the split-K arrival counters must come back reset
        y.zero_()
        sq.linear_w8a8(dev(A), dev(B), dev(a), mode, dev(ws), y,
                       bias=dev(bias, out_dt) if with_bias else None, workspace=work)
        _sync()
        ref = oracle.dequant(acc_ref, a, mode, ws, out_dt, bias)
        got = host(y)
        assert bits_equal(got, ref), mismatch_report(got, ref)


@pytest.fixture
def _no_cluster_split():
    sq.lib().sq_debug_inject(2)
    try:
        yield
    finally:
        sq.lib().sq_debug_inject(0)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 11008), (16, 4096, 4096), (5, 1024, 4112), (32, 2048, 8192),
                                   (17, 4096, 11008), (3, 256, 65536), (1, 11008, 4096), (33, 11008, 4112),
                                   (100, 4096, 4096), (128, 18944, 256), (64, 1040, 528), (128, 2048, 11008)])
@pytest.mark.parametrize("schedule", ["cluster", "stream_k"])
def test_linear_w8a8_small_m_schedules(M, N, K, schedule, request):
    """Small-M path on its schedules -- the cluster split (2 or 4 CTAs per
    weight tile, partial sums combined in distributed shared memory) and,
    with the cluster split off, the stream-K schedule with a workspace --
    against the one-tile-per-CTA launch, bit for bit, twice (the stream-K
    arrival counters must come back reset), and against the oracle on
    sampled output channels (first, last and random rows of W)."""
    if schedule == "stream_k":
        request.getfixturevalue("_no_cluster_split")
    g = np.random.default_rng(M * 5 + N + K)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (N, K), dtype=np.int8)
    a = (np.abs(g.standard_normal(M)) * 1e-2 + 1e-3).astype(np.float32)
    ws = (np.abs(g.standard_normal(N)) * 1e-4 + 1e-5).astype(np.float32)
    bias = synth.cast(g.standard_normal(N).astype(np.float32), BF16)
    dA, dB, da, dws, db = dev(A), dev(B), dev(a), dev(ws), dev(bias, BF16)
    y0 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    hook = 2 if schedule == "stream_k" else 0
    sq.lib().sq_debug_inject(2)                     # reference: one tile per CTA (no workspace)
    sq.linear_w8a8(dA, dB, da, oracle.PER_TOKEN, dws, y0, bias=db)
    _sync()
    sq.lib().sq_debug_inject(hook)
    n = sq.linear_workspace_size(M, N, K)
    work = torch.zeros(max(16, n), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        sq.linear_w8a8(dA, dB, da, oracle.PER_TOKEN, dws, y, bias=db, workspace=work)
        _sync()
        assert torch.equal(y.view(torch.int16), y0.view(torch.int16))
    idx = np.unique(np.concatenate([np.arange(min(N, 160)), np.arange(max(0, N - 160), N),
                                    g.integers(0, N, 64)]))
    acc = oracle.gemm_s32(A, B[idx])
    ref = oracle.dequant(acc, a, oracle.PER_TOKEN, ws[idx], BF16, bias[idx])
    got = host(y)[:, idx]
    assert bits_equal(got, ref), mismatch_report(got, ref)


@pytest.mark.parametrize("M,N,K", [(96, 11008, 4096), (80, 9728, 4112), (65, 12288, 2048), (100, 11008, 528),
                                   (128, 19456, 4096), (128, 9600, 11008)])
@pytest.mark.parametrize("out_dt,mode", [(BF16, oracle.PER_TOKEN), (F16, oracle.STATIC), (F32, oracle.PER_TOKEN)])
def test_linear_w8a8_pair_swapped(M, N, K, out_dt, mode):
    """64 < M <= 128 with many weight rows runs the CTA-pair kernel with the
    weights as its A operand and the tokens as B (transposed epilogue):
    bit-identical to the weight-streaming schedule (sq_debug_inject(2)) and
    to the oracle on sampled output channels, with bias, per-token and static
    scales, K a multiple of 128 and not, ragged token and channel tiles."""
    g = np.random.default_rng(M * 11 + N + K)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (N, K), dtype=np.int8)
    a = (np.abs(g.standard_normal(1 if mode == oracle.STATIC else M)) * 1e-2 + 1e-3).astype(np.float32)
    ws = (np.abs(g.standard_normal(N)) * 1e-4 + 1e-5).astype(np.float32)
    bias = synth.cast(g.standard_normal(N).astype(np.float32), out_dt) if out_dt != F32 else None
    dA, dB, da, dws = dev(A), dev(B), dev(a), dev(ws)
    db = dev(bias, out_dt) if bias is not None else None
    torch_dt = {BF16: torch.bfloat16, F16: torch.float16, F32: torch.float32}[out_dt]
    y0 = torch.empty(M, N, dtype=torch_dt, device="cuda")
    sq.lib().sq_debug_inject(2)
    try:
        sq.linear_w8a8(dA, dB, da, mode, dws, y0, bias=db)
        _sync()
    finally:
        sq.lib().sq_debug_inject(0)
    y = torch.full((M, N), float("nan"), dtype=torch_dt, device="cuda")
    sq.linear_w8a8(dA, dB, da, mode, dws, y, bias=db)
    _sync()
    iv = torch.int32 if out_dt == F32 else torch.int16
    assert torch.equal(y.view(iv), y0.view(iv))
    idx = np.unique(np.concatenate([np.arange(160), np.arange(N - 160, N), g.integers(0, N, 64)]))
    ref = oracle.dequant(oracle.gemm_s32(A, B[idx]), a, mode, ws[idx], out_dt,
                         bias[idx] if bias is not None else None)
    assert bits_equal(host(y)[:, idx], ref), mismatch_report(host(y)[:, idx], ref)


# ------------------------------------------------------------------ a9
@pytest.mark.parametrize("M,Nh,K", [(300, 256, 512), (129, 384, 1040)])
def test_gateup_silu(M, Nh, K):
    g = np.random.default_rng(M + Nh)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    Bg = g.integers(-127, 128, (Nh, K), dtype=np.int8)
    Bu = g.integers(-127, 128, (Nh, K), dtype=np.int8)
    a = np.array([2e-3], np.float32)
    wsg = (np.abs(g.standard_normal(Nh)) * 1e-3 + 1e-4).astype(np.float32)
    wsu = (np.abs(g.standard_normal(Nh)) * 1e-3 + 1e-4).astype(np.float32)
    order = np.concatenate([np.concatenate([np.arange(b, b + 32), Nh + np.arange(b, b + 32)])
                            for b in range(0, Nh, 32)])
    Bgu = np.concatenate([Bg, Bu])[order]
    wsgu = np.concatenate([wsg, wsu])[order]
    s2 = (np.abs(g.standard_normal(Nh)) + 0.5).astype(np.float32)
    a2 = np.array([0.02], np.float32)
    h = torch.empty(M, Nh, dtype=torch.bfloat16, device="cuda")
    hq = torch.empty(M, Nh, dtype=torch.int8, device="cuda")
    sq.linear_w8a8_gateup_silu(dev(A), dev(Bgu), dev(a), oracle.STATIC, dev(wsgu), h=h, s2=dev(s2),
                               a2=dev(a2), hq=hq)
    _sync()
    gv = oracle.dequant_f32(oracle.gemm_s32(A, Bg), a, oracle.STATIC, wsg)
    uv = oracle.dequant_f32(oracle.gemm_s32(A, Bu), a, oracle.STATIC, wsu)
    h_ref = oracle.silu_mul_bf16(gv, uv)
    h_got = host(h)
    hf_got = oracle.to_f32(h_got, BF16).astype(np.float64)
    hf_ref = oracle.to_f32(h_ref, BF16).astype(np.float64)
    ulp = np.maximum(np.abs(hf_ref), 1e-30) * 2.0 ** -7
    assert np.all(np.abs(hf_got - hf_ref) <= 2 * ulp + 1e-30)
    assert (h_got != h_ref).mean() < 0.01
    # requantised h: exactly the oracle's codes wherever h agrees bitwise
    hq_ref, _ = oracle.smooth_quant_act(h_ref, s2, oracle.STATIC, a2[0], BF16)
    hq_got = host(hq)
    same = h_got == h_ref
    assert np.array_equal(hq_got[same], hq_ref[same])
    assert np.all(np.abs(hq_got.astype(int) - hq_ref.astype(int)) <= 1)
    # the h-only and hq-only forms agree with the combined one
    h2 = torch.empty_like(h)
    sq.linear_w8a8_gateup_silu(dev(A), dev(Bgu), dev(a), oracle.STATIC, dev(wsgu), h=h2)
    hq2 = torch.empty_like(hq)
    sq.linear_w8a8_gateup_silu(dev(A), dev(Bgu), dev(a), oracle.STATIC, dev(wsgu), s2=dev(s2), a2=dev(a2), hq=hq2)
    _sync()
    assert torch.equal(h2.view(torch.int16), h.view(torch.int16)) and torch.equal(hq2, hq)


# ------------------------------------------------------------------ a7
@pytest.mark.parametrize("M,N,K", [(200, 272, 520), (64, 512, 1024)])
def test_gemm_f16_ref(M, N, K):
    X = rand_x(M, (M, K), F16, 1.0)
    W = rand_x(N, (N, K), F16, 0.05)
    y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    sq.gemm_f16_ref(dev(X, F16), dev(W, F16), y)
    _sync()
    ref = oracle.gemm_f16_ref(X, W)
    got = oracle.to_f32(host(y), F16).astype(np.float64)
    want = oracle.to_f32(ref, F16).astype(np.float64)
    # fp32 accumulation (order differs from the fp64 sum) + one fp16 rounding
    mag = np.abs(oracle.to_f32(X, F16).astype(np.float64)) @ np.abs(oracle.to_f32(W, F16).astype(np.float64)).T
    tol = np.abs(want) * 2.0 ** -10 + mag * K * 2.0 ** -24 + 2.0 ** -24
    assert np.all(np.abs(got - want) <= tol)


def test_sse_f16():
    g = np.random.default_rng(0)
    y = g.standard_normal(100003).astype(np.float16)
    r = g.standard_normal(100003).astype(np.float16)
    sse = torch.zeros(1, dtype=torch.float64, device="cuda")
    yt = torch.from_numpy(y).cuda()
    rt = torch.from_numpy(r).cuda()
    sq.sse_f16(yt, rt, sse)
    _sync()
    ref = oracle.mse_f16(y.view(np.uint16), r.view(np.uint16)) * y.size
    assert abs(float(sse.item()) - ref) <= 1e-9 * ref


def test_alpha_search_small():
    wl = synth.heavy_13b(M=64, K=512, N=272, calib_batches=4, calib_rows=128)
    am = np.zeros(wl.K, np.float32)
    for b in wl.calib:
        oracle.calib_absmax(b, F16, am)
    wm = oracle.calib_absmax(wl.w, F16)
    best_ref, mse_ref, _ = oracle.alpha_search(wl.calib[0], wl.w, am, wm)
    held = wl.calib[0]
    work = torch.zeros(sq.alpha_search_workspace_size(held.shape[0], wl.N, wl.K, 4), dtype=torch.uint8,
                       device="cuda")
    best, mses = sq.alpha_search(dev(held, F16), dev(wl.w, F16), dev(am), dev(wm), work)
    assert best == best_ref
    assert rel_err(mses, mse_ref).max() < 1e-4


# ------------------------------------------------------------------ a8 statistic
@pytest.mark.parametrize("M,d,dt", [(300, 8192, BF16), (7, 4096, F16), (33, 1000, BF16), (5, 2048, F32),
                                    (3, 11008, BF16)])
def test_rmsnorm_absmax(M, d, dt):
    X = rand_x(M * 5 + d, (M, d), dt, 1.0, outliers=max(1, d // 200))
    gamma = np.random.default_rng(d + 1).uniform(0.5, 1.5, d).astype(np.float32)
    am = torch.zeros(d, dtype=torch.float32, device="cuda")
    half = M // 2
    xt = dev(X, dt)
    sq.rmsnorm_absmax(xt[:half] if half else xt[:0], dev(gamma), 1e-5, am)
    sq.rmsnorm_absmax(xt[half:], dev(gamma), 1e-5, am)
    _sync()
    ref = oracle.rmsnorm_absmax(X, gamma, 1e-5, dt)
    assert bits_equal(host(am), ref), mismatch_report(host(am), ref)


@pytest.mark.parametrize("M,K,dt", [(5000, 8192, BF16), (9001, 4096, F16), (3001, 6144, BF16), (2000, 3000, BF16),
                                    (1500, 1032, F16)])
def test_rmsnorm_many_rows_per_block(M, K, dt):
    """RMSNorm + quant and the norm-output statistic with many rows per block
    (each block walks rows with the next row's loads in flight; the
    statistic's rows come through the shared-memory row ring), at row counts
    that are not a multiple of the grid and row lengths with a ragged last
    vector group, bit for bit against the oracle."""
    X = rand_x(M + K + 3, (M, K), dt, 1.0, outliers=max(1, K // 200))
    g = np.random.default_rng(M * 3 + K)
    gamma = g.uniform(0.5, 1.5, K).astype(np.float32)
    s = (np.abs(g.standard_normal(K)) + 0.3).astype(np.float32)
    a = np.float32(0.04)
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    r = torch.empty(M, dtype=torch.float32, device="cuda")
    xt = dev(X, dt)
    sq.rmsnorm_quant(xt, dev(gamma), dev(s), 1e-5, dev(np.array([a])), xq, r)
    am = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.rmsnorm_absmax(xt, dev(gamma), 1e-5, am)
    _sync()
    xq_ref, r_ref = oracle.rmsnorm_quant(X, gamma, s, 1e-5, a, dt)
    assert bits_equal(host(r), r_ref), mismatch_report(host(r), r_ref)
    assert bits_equal(host(xq), xq_ref), mismatch_report(host(xq), xq_ref)
    am_ref = oracle.rmsnorm_absmax(X, gamma, 1e-5, dt)
    assert bits_equal(host(am), am_ref), mismatch_report(host(am), am_ref)


# ------------------------------------------------------------------ row ring
@pytest.mark.parametrize("case", ["token_bf16_8192", "token_f16_6144", "token_f32_8192", "weight_bf16_8192",
                                  "gateup_bf16_8192", "stat_bf16_4096", "stat_f16_8192"])
def test_row_ring_paths(case):
    """Row kernels whose rows come through the shared-memory ring of bulk
    copies (256-thread rows held in registers: per-token quant and the weight
    transform; the norm-output statistic from 64 rows per SM up), at row
    counts that are not a multiple of the grid and with a ragged last vector
    group (6144 = 3 vectors per thread of 4), bit for bit against the oracle."""
    kind, dname, k = case.split("_")
    dt = {"bf16": BF16, "f16": F16, "f32": F32}[dname]
    K = int(k)
    g = np.random.default_rng(K + len(case))
    s = (np.abs(g.standard_normal(K)) + 0.2).astype(np.float32)
    if kind == "token":
        M = 1000 if dt != F32 else 400
        X = rand_x(M + K, (M, K), dt, 2.0, outliers=8)
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        at = torch.empty(M, dtype=torch.float32, device="cuda")
        sq.smooth_quant_act(dev(X, dt), dev(s), oracle.PER_TOKEN, at, xq)
        _sync()
        xq_ref, a_ref = oracle.smooth_quant_act(X, s, oracle.PER_TOKEN, None, dt)
        assert bits_equal(host(at), a_ref), mismatch_report(host(at), a_ref)
        assert bits_equal(host(xq), xq_ref), mismatch_report(host(xq), xq_ref)
    elif kind == "weight":
        N = 1000
        W = rand_x(N + K, (N, K), dt, 0.02)
        wq = torch.empty(N, K, dtype=torch.int8, device="cuda")
        ws = torch.empty(N, dtype=torch.float32, device="cuda")
        sq.quant_weight(dev(W, dt), dev(s), wq, ws)
        _sync()
        wq_ref, ws_ref = oracle.quant_weight(W, s, dt)
        assert bits_equal(host(ws), ws_ref), mismatch_report(host(ws), ws_ref)
        assert bits_equal(host(wq), wq_ref), mismatch_report(host(wq), wq_ref)
    elif kind == "gateup":
        Nh = 160
        Wg = rand_x(11, (Nh, K), dt, 0.02)
        Wu = rand_x(12, (Nh, K), dt, 0.02)
        wq = torch.empty(2 * Nh, K, dtype=torch.int8, device="cuda")
        ws = torch.empty(2 * Nh, dtype=torch.float32, device="cuda")
        sq.quant_weight_gateup(dev(Wg, dt), dev(Wu, dt), dev(s), wq, ws)
        _sync()
        order = np.concatenate([np.concatenate([np.arange(b, b + 32), Nh + np.arange(b, b + 32)])
                                for b in range(0, Nh, 32)])
        wq_ref, ws_ref = oracle.quant_weight(np.concatenate([Wg, Wu])[order], s, dt)
        assert bits_equal(host(wq), wq_ref) and bits_equal(host(ws), ws_ref)
    else:
        M = 9500 if K == 4096 else 9600          # >= 64 rows per SM of a 148-SM part: ring path
        X = rand_x(M + K, (M, K), dt, 1.0, outliers=max(1, K // 200))
        gamma = g.uniform(0.5, 1.5, K).astype(np.float32)
        am = torch.zeros(K, dtype=torch.float32, device="cuda")
        sq.rmsnorm_absmax(dev(X, dt), dev(gamma), 1e-5, am)
        _sync()
        ref = oracle.rmsnorm_absmax(X, gamma, 1e-5, dt)
        assert bits_equal(host(am), ref), mismatch_report(host(am), ref)


@pytest.mark.parametrize("dt", [F32, BF16])
def test_quant_tiny_rows_saturate_like_the_oracle(dt):
    """Rows whose max gives a subnormal scale: codes still clamp to +-127 like the oracle's."""
    K = 512
    W = np.zeros((4, K), np.float32)
    W[0, :] = 1e-39
    W[0, 7] = -3e-39
    W[1, 3] = 1e-44
    W[2, :] = np.linspace(-1, 1, K)
    Wd = synth.cast(W, dt)
    s = np.ones(K, np.float32)
    wq = torch.empty(4, K, dtype=torch.int8, device="cuda")
    ws = torch.empty(4, dtype=torch.float32, device="cuda")
    sq.quant_weight(dev(Wd, dt), dev(s), wq, ws)
    xq = torch.empty(4, K, dtype=torch.int8, device="cuda")
    at = torch.empty(4, dtype=torch.float32, device="cuda")
    sq.smooth_quant_act(dev(Wd, dt), dev(s), oracle.PER_TOKEN, at, xq)
    _sync()
    wq_r, ws_r = oracle.quant_weight(Wd, s, dt)
    xq_r, a_r = oracle.smooth_quant_act(Wd, s, oracle.PER_TOKEN, None, dt)
    assert bits_equal(host(ws), ws_r) and bits_equal(host(at), a_r)
    assert np.array_equal(host(wq), wq_r), mismatch_report(host(wq), wq_r)
    assert np.array_equal(host(xq), xq_r), mismatch_report(host(xq), xq_r)
