"""Failure detection without a GPU fault: a GEMM whose pipeline stage is
withheld (test hook) must give up its bounded barrier wait, report
SQ_ERR_TIMEOUT through sq_sync_status, and leave the CUDA context usable."""
import numpy as np
import pytest
import torch

import oracle
from helpers import dev, host

pytestmark = pytest.mark.gpu

sq = pytest.importorskip("w8a8_post_quantization_calib_b200")


@pytest.mark.parametrize("M,N,K", [(16, 512, 1024), (300, 768, 1024)])   # small-M path, CTA-pair path
def test_withheld_stage_times_out_and_context_survives(M, N, K):
    g = np.random.default_rng(M)
    A = g.integers(-127, 128, (M, K), dtype=np.int8)
    B = g.integers(-127, 128, (N, K), dtype=np.int8)
    acc = torch.zeros(M, N, dtype=torch.int32, device="cuda")
    assert sq.sync_status() == 0
    sq.set_wait_timeout_ns(20_000_000)          # 20 ms per barrier wait
    sq.lib().sq_debug_inject(1)
    try:
        sq.gemm_s32(dev(A), dev(B), acc)         # launches fine; the kernel gives up inside
        assert sq.sync_status() == 5             # SQ_ERR_TIMEOUT, reported once ...
        assert sq.sync_status() == 0             # ... and cleared
    finally:
        sq.lib().sq_debug_inject(0)
        sq.set_wait_timeout_ns(0)
    sq.gemm_s32(dev(A), dev(B), acc)
    assert sq.sync_status() == 0
    assert np.array_equal(host(acc), oracle.gemm_s32(A, B))
