"""sq_linear_w8a8_noalloc against sq_linear_w8a8 (GPU).

sq_linear_w8a8_noalloc is the W8A8 linear for callers that cannot allocate
device memory (a plugin that only receives its input and output buffers from
a host engine, or a serving loop that must not pay cudaMalloc's device-wide
synchronisation).  It takes no workspace: its small-M split-K path keeps the
partial sums in a fixed array inside the library.  This file checks, through
the C ABI, that it returns exactly what the workspace-taking entry point
returns, on two calls in a row (the second call finds the first call's
leftovers in the shared array), after a call of another shape and after a
call that timed out, and that oversize requests are refused before any
launch.  It is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

sq = pytest.importorskip("w8a8_post_quantization_calib_b200")

_OUT = {0: torch.float32, 1: torch.float16, 2: torch.bfloat16}


def _operands(M, N, K, mode, out_dt, seed):
    g = np.random.default_rng(seed)
    xq = torch.from_numpy(g.integers(-127, 128, (M, K), dtype=np.int8)).cuda()
    wq = torch.from_numpy(g.integers(-127, 128, (N, K), dtype=np.int8)).cuda()
    a = torch.from_numpy((np.abs(g.standard_normal(1 if mode == 0 else M)) * 1e-2 + 1e-3).astype(np.float32)).cuda()
    ws = torch.from_numpy((np.abs(g.standard_normal(N)) * 1e-4 + 1e-5).astype(np.float32)).cuda()
    bias = torch.from_numpy(g.standard_normal(N).astype(np.float32)).cuda().to(_OUT[out_dt])
    return xq, wq, a, ws, bias


def _call_noalloc(xq, wq, a, mode, ws, bias, y):
    M, K = xq.shape
    N = wq.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    return sq.lib().sq_linear_w8a8_noalloc(
        xq.data_ptr(), wq.data_ptr(), M, N, K, a.data_ptr(), mode, ws.data_ptr(),
        bias.data_ptr() if bias is not None else None, {torch.float32: 0, torch.float16: 1,
                                                        torch.bfloat16: 2}[y.dtype],
        y.data_ptr(), stream)


def _call_with_workspace(xq, wq, a, mode, ws, bias, y):
    M, K = xq.shape
    N = wq.shape[0]
    n = sq.lib().sq_linear_workspace_size(M, N, K)
    work = torch.zeros(max(n, 16), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = sq.lib().sq_linear_w8a8(
        xq.data_ptr(), wq.data_ptr(), M, N, K, a.data_ptr(), mode, ws.data_ptr(),
        bias.data_ptr() if bias is not None else None, {torch.float32: 0, torch.float16: 1,
                                                        torch.bfloat16: 2}[y.dtype],
        y.data_ptr(), work.data_ptr(), n, stream)
    return st


@pytest.fixture(params=[0, 2], ids=["cluster_split", "stream_k_scratch"])
def _hook(request):
    """0: default schedules (the small-M cluster split needs no scratch);
    2: cluster split off, so the small-M path shares tiles through the
    library's fixed scratch array."""
    sq.lib().sq_debug_inject(request.param)
    try:
        yield request.param
    finally:
        sq.lib().sq_debug_inject(0)


@pytest.mark.parametrize("M,N,K,mode,out_dt,with_bias", [
    (16, 4096, 11008, 1, 2, False),     # decode-size down projection: tiles shared across CTAs
    (1, 11008, 4096, 1, 2, True),
    (64, 2048, 1024, 0, 1, True),
    (128, 1024, 4096, 0, 0, False),
    (100, 11008, 4096, 1, 2, True),     # swapped CTA pairs (64 < M <= 128, many weight rows)
    (300, 528, 1040, 1, 1, True),       # large M: no scratch needed
])
def test_noalloc_matches_workspace_entry_point(M, N, K, mode, out_dt, with_bias, _hook):
    xq, wq, a, ws, bias = _operands(M, N, K, mode, out_dt, M * 31 + N)
    bias = bias if with_bias else None
    y_ref = torch.empty(M, N, dtype=_OUT[out_dt], device="cuda")
    assert _call_with_workspace(xq, wq, a, mode, ws, bias, y_ref) == 0
    for _ in range(2):                  # two calls in a row share the library's array
        y = torch.full((M, N), float("nan"), dtype=_OUT[out_dt], device="cuda")
        assert _call_noalloc(xq, wq, a, mode, ws, bias, y) == 0
        assert sq.sync_status() == 0
        # same kernel, same exact int32 sums, same epilogue: bit-identical
        assert torch.equal(y.view(torch.uint8), y_ref.view(torch.uint8))


def test_noalloc_back_to_back_different_shapes(_hook):
    """A smaller call after a larger one must not see the larger call's leftovers.

    With the cluster split off both shapes share weight tiles between CTAs,
    i.e. both go through the library's array (the workspace entry point asks
    for a workspace exactly when its schedule shares tiles, and the no-alloc
    entry point runs the same schedule)."""
    big = _operands(32, 8192, 4096, 1, 2, 1)          # 64 weight tiles, 32-token tile
    small = _operands(16, 1024, 4096, 1, 2, 2)        # 8 weight tiles
    if _hook == 2:
        for ops in (big, small):
            M, N, K = ops[0].shape[0], ops[1].shape[0], ops[0].shape[1]
            assert sq.lib().sq_linear_workspace_size(M, N, K) > 0
    outs = []
    for ops in (big, small, big):
        xq, wq, a, ws, _ = ops
        y_ref = torch.empty(xq.shape[0], wq.shape[0], dtype=torch.bfloat16, device="cuda")
        assert _call_with_workspace(xq, wq, a, 1, ws, None, y_ref) == 0
        y = torch.empty_like(y_ref)
        assert _call_noalloc(xq, wq, a, 1, ws, None, y) == 0
        outs.append((y, y_ref))
    assert sq.sync_status() == 0
    for y, y_ref in outs:
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))


def test_noalloc_rejects_oversize_without_launch():
    """A request whose tile-sharing schedule needs more partial-sum slots than
    the array holds is refused before anything runs.  No B200 request is that
    large (one 128 x 16 int32 slot per CTA, 148 CTAs: 1.2 MB here), so the
    test hook 4 makes the size check assume a 64 KiB array."""
    assert sq.lib().sq_linear_w8a8_noalloc_max_elems() == 2 ** 21
    M, N, K = 16, 4096, 11008
    xq, wq, a, ws, _ = _operands(M, N, K, 1, 1, 5)
    sq.lib().sq_debug_inject(2 | 4)
    try:
        assert sq.lib().sq_linear_workspace_size(M, N, K) > 64 * 1024    # the schedule shares tiles
        y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
        assert _call_noalloc(xq, wq, a, 1, ws, None, y) == 2             # SQ_ERR_UNSUPPORTED
        assert sq.sync_status() == 0
        assert torch.all(y == 7.0)                                        # nothing was launched
        # a shape whose schedule keeps its partial sums on chip is never refused,
        # whatever its size (M*N here is 2.5 M values)
        M2, N2, K2 = 128, 20480, 256
        xq2, wq2, a2, ws2, _ = _operands(M2, N2, K2, 0, 2, 6)
        assert sq.lib().sq_linear_workspace_size(M2, N2, K2) == 0
        y_ref = torch.empty(M2, N2, dtype=torch.bfloat16, device="cuda")
        assert _call_with_workspace(xq2, wq2, a2, 0, ws2, None, y_ref) == 0
        y2 = torch.full((M2, N2), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(xq2, wq2, a2, 0, ws2, None, y2) == 0
        assert sq.sync_status() == 0
        assert torch.equal(y2.view(torch.int16), y_ref.view(torch.int16))
    finally:
        sq.lib().sq_debug_inject(0)


def test_noalloc_after_a_timed_out_call():
    """A call whose bounded wait ran out leaves tile counters raised in the
    array; the next call clears the counters it uses and is exact again."""
    M, N, K = 16, 4096, 11008
    xq, wq, a, ws, _ = _operands(M, N, K, 1, 2, 9)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    assert sq.sync_status() == 0
    sq.set_wait_timeout_ns(20_000_000)                  # 20 ms per barrier wait
    sq.lib().sq_debug_inject(1 | 2)                     # withheld stage, stream-K schedule
    try:
        assert sq.lib().sq_linear_workspace_size(M, N, K) > 0
        assert _call_noalloc(xq, wq, a, 1, ws, None, y) == 0           # launches; gives up inside
        assert sq.sync_status() == 5                                    # SQ_ERR_TIMEOUT
        sq.lib().sq_debug_inject(2)
        y_ref = torch.empty_like(y)
        assert _call_with_workspace(xq, wq, a, 1, ws, None, y_ref) == 0
        y.fill_(float("nan"))
        assert _call_noalloc(xq, wq, a, 1, ws, None, y) == 0
        assert sq.sync_status() == 0
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    finally:
        sq.lib().sq_debug_inject(0)
        sq.set_wait_timeout_ns(0)
