"""Robust calibration statistics on the GPU against the oracle (kwkr.cn blog
3.1: a 99.9 % quantile of |X_j|, or the mean of the calibration samples'
maxima, in place of the max).  Both results are exact functions of the data
(a data value; an fp64 sum in sample order rounded once), so the GPU and the
oracle agree bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import BF16, F16, F32, bits_equal, dev, host, mismatch_report, rand_x

pytestmark = pytest.mark.gpu

sq = pytest.importorskip("w8a8_post_quantization_calib_b200")


def _sync():
    assert sq.sync_status() == 0


def _quantile(x_bits, dt, p, ld_pad=0):
    T, K = x_bits.shape
    if ld_pad:
        wide = np.zeros((T, K + ld_pad), x_bits.dtype)
        wide[:, :K] = x_bits
        xt = dev(wide, dt)[:, :K]
    else:
        xt = dev(x_bits, dt)
    out = torch.full((K,), -1.0, dtype=torch.float32, device="cuda")
    work = torch.empty(sq.calib_quantile_workspace_size(K), dtype=torch.uint8, device="cuda")
    sq.calib_quantile(xt, p, out, work)
    _sync()
    return host(out)


@pytest.mark.parametrize("T,K,dt", [(2048, 4096, F16), (777, 1000, BF16), (300, 520, F32), (1, 256, F16),
                                    (4096, 136, BF16)])
@pytest.mark.parametrize("p", [1.0, 0.999, 0.9, 0.5, 1e-9])
def test_quantile_matches_oracle(T, K, dt, p):
    X = rand_x(T * 7 + K, (T, K), dt, 1.0, outliers=max(1, K // 200))
    got = _quantile(X, dt, p)
    want = oracle.calib_quantile([X], p, dt)
    assert bits_equal(got, want), mismatch_report(got, want)


def test_quantile_one_is_the_max_and_strided_rows():
    X = rand_x(11, (1500, 1024), BF16, 3.0, outliers=5)
    got = _quantile(X, BF16, 1.0, ld_pad=64)              # rows 1088 elements apart
    am = torch.zeros(1024, dtype=torch.float32, device="cuda")
    sq.calib_absmax(dev(X, BF16), am)
    _sync()
    assert bits_equal(got, host(am))


def test_quantile_ties_and_special_values():
    """Many equal magnitudes (ties of rank), signed zeros, subnormals and the
    largest finite values: the selected value is still the oracle's."""
    g = np.random.default_rng(3)
    T, K = 1000, 256
    vals = np.array([0.0, -0.0, 1.0, -1.0, 2.0 ** -24, -(2.0 ** -24), 65504.0, -65504.0, 0.5, 3.0], np.float32)
    X = synth.cast(vals[g.integers(0, len(vals), (T, K))], F16)
    for p in (1.0, 0.999, 0.75, 0.5, 0.3, 0.001):
        got = _quantile(X, F16, p)
        want = oracle.calib_quantile([X], p, F16)
        assert bits_equal(got, want), (p, mismatch_report(got, want))


def test_quantile_ignores_a_planted_outlier():
    """kwkr.cn 3.1: one abnormal token moves the max but not the 99.9 % quantile."""
    wl = synth.qkv_7b(M=16, K=512, N=64, calib_batches=16, calib_rows=512)
    X = np.concatenate(wl.calib)                    # 8192 tokens: the 99.9 % rank is the 9th largest
    Xo = X.copy()
    Xo[1234] = synth.cast(np.full(512, 5000.0, np.float32), F16)
    q_clean, q_out = _quantile(X, F16, 0.999), _quantile(Xo, F16, 0.999)
    m_out = _quantile(Xo, F16, 1.0)
    assert np.all(m_out == 5000.0)
    assert bits_equal(q_out, oracle.calib_quantile([Xo], 0.999, F16))
    # one token moves the rank by one place among the largest values: the
    # statistic moves a little, the max by orders of magnitude
    assert np.max(q_out / np.maximum(q_clean, 1e-30)) <= 1.25
    assert np.max(q_out) < 5000.0 / 10


@pytest.mark.parametrize("dt", [F16, BF16, F32])
def test_mean_of_max_matches_oracle(dt):
    K = 1000 if dt != F32 else 520
    batches = [rand_x(100 + b, (64 + 17 * b, K), dt, 1.0 + b, outliers=3) for b in range(6)]
    bm = torch.zeros(K, dtype=torch.float32, device="cuda")
    acc = torch.zeros(K, dtype=torch.float64, device="cuda")
    for b in batches:
        sq.calib_batchmax_accumulate(dev(b, dt), bm, acc)
    out = torch.empty(K, dtype=torch.float32, device="cuda")
    sq.calib_mean_of_max(acc, len(batches), out)
    _sync()
    want = oracle.calib_mean_of_max(batches, dt)
    assert bits_equal(host(out), want), mismatch_report(host(out), want)
    assert np.all(host(bm) == 0.0)                        # the scratch is left zero


def test_robust_statistic_feeds_the_smoothing_factors():
    """The 99.9 % statistic of the QKV calibration set stands in for act_max:
    s from the GPU statistic equals the oracle's s from the oracle statistic
    within 1e-6 relative."""
    wl = synth.qkv_7b(M=16, K=4096, N=256, calib_batches=8, calib_rows=512)
    X = np.concatenate(wl.calib)
    q = _quantile(X, F16, 0.999)
    wm = oracle.calib_absmax(wl.w, F16)
    s = torch.empty(4096, dtype=torch.float32, device="cuda")
    sq.smooth_scales(dev(q), dev(wm), 0.5, s)
    _sync()
    s_r = oracle.smooth_scales(oracle.calib_quantile([X], 0.999, F16), wm, 0.5)
    assert np.max(np.abs(host(s) / s_r - 1)) <= 1e-6
