"""The C ABI library loads and exports every entry point declared in include/sq.h (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "sq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_five_core_calls():
    names = _declared()
    for core in ("sq_calib_absmax", "sq_smooth_scales", "sq_quant_weight", "sq_smooth_quant_act",
                 "sq_linear_w8a8"):
        assert core in names


def test_library_exports_every_declared_symbol():
    from w8a8_post_quantization_calib_b200 import LIB_PATH, EXPORTS
    lib = ctypes.CDLL(LIB_PATH)
    names = _declared()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(EXPORTS) == names          # the binding wraps exactly the declared calls


def test_measurement_library_loads_and_exports_its_calls():
    """libsq_peak.so (the tensor-core peak and streaming-read ceiling used as
    roofline denominators) loads without a GPU and exports its calls; the
    streaming read validates its arguments before launching."""
    from w8a8_post_quantization_calib_b200 import peak
    lib = peak.lib()
    for name in ("sqpeak_clusters", "sqpeak_launch", "sqpeak_error_word", "sqpeak_stream_read"):
        assert hasattr(lib, name), name
    inval = 1                                    # cudaErrorInvalidValue
    assert lib.sqpeak_stream_read(None, 16, 1, None, None) == inval
    assert lib.sqpeak_stream_read(16, 15, 1, None, None) == inval        # bytes not a multiple of 16
    assert lib.sqpeak_stream_read(8, 16, 1, None, None) == inval         # misaligned
    assert lib.sqpeak_stream_read(16, 16, 0, None, None) == inval        # no blocks
    assert lib.sqpeak_launch(0, 0, 1, None) == inval
    assert lib.sqpeak_launch(0, 1, (1 << 20) + 1, None) == inval


def test_host_only_entry_points_without_gpu():
    import w8a8_post_quantization_calib_b200 as sq
    lib = sq.lib()
    assert lib.sq_status_string(0) == b"SQ_OK"
    assert lib.sq_status_string(5) == b"SQ_ERR_TIMEOUT"
    # sizes are pure host arithmetic
    # the small-M cluster split combines partial sums on chip: no workspace
    assert sq.linear_workspace_size(16, 4096, 11008) == 0
    assert sq.linear_workspace_size(4096, 4096, 11008) == 0
    lib.sq_debug_inject(2)                   # cluster split off: stream-K slots + counters
    try:
        assert sq.linear_workspace_size(16, 4096, 11008) >= 16 * 4096 * 4
    finally:
        lib.sq_debug_inject(0)
    assert sq.alpha_search_workspace_size(512, 13824, 5120, 4) > 13824 * 5120


@pytest.mark.parametrize("args", [
    dict(rows=-1), dict(cols=0), dict(ld=3), dict(dt=7),
])
def test_argument_validation_rejects_without_launch(args):
    """Bad arguments return SQ_ERR_INVALID_ARG before any CUDA call (safe without a GPU)."""
    import w8a8_post_quantization_calib_b200 as sq
    lib = sq.lib()
    kw = dict(x=16, dt=1, rows=4, cols=8, ld=8, absmax=32)
    kw.update(args)
    st = lib.sq_calib_absmax(kw["x"], kw["dt"], kw["rows"], kw["cols"], kw["ld"], kw["absmax"], None)
    assert st == 1


def test_gemm_validation():
    import w8a8_post_quantization_calib_b200 as sq
    lib = sq.lib()
    # N not a multiple of 16, K not a multiple of 16, null pointers, misaligned operands
    assert lib.sq_linear_w8a8(16, 16, 4, 24, 64, 16, 0, 16, None, 1, 16, None, 0, None) == 1
    assert lib.sq_linear_w8a8(16, 16, 4, 32, 40, 16, 0, 16, None, 1, 16, None, 0, None) == 1
    assert lib.sq_linear_w8a8(None, 16, 4, 32, 64, 16, 0, 16, None, 1, 16, None, 0, None) == 1
    assert lib.sq_linear_w8a8(17, 16, 4, 32, 64, 16, 0, 16, None, 1, 16, None, 0, None) == 3
    assert lib.sq_smooth_scales(16, 16, 8, 1.5, 16, None, None) == 1
    assert lib.sq_smooth_scales(16, 16, 8, -0.1, 16, None, None) == 1


# Every entry point validates its arguments on the host and returns before
# any CUDA call, so these run without a GPU.  Pointers are fake addresses
# (16 = aligned, 17 = misaligned); no call below reaches a launch.
_A, _U = 16, 17


def _alphas(*v):
    import ctypes
    return (ctypes.c_float * len(v))(*v)


@pytest.mark.parametrize("fn,args,status", [
    ("sq_quant_weight", (None, 1, 8, 64, _A, _A, _A, None), 1),
    ("sq_quant_weight", (_A, 9, 8, 64, _A, _A, _A, None), 1),
    ("sq_quant_weight", (_A, 1, -1, 64, _A, _A, _A, None), 1),
    ("sq_quant_weight", (_U, 1, 8, 64, _A, _A, _A, None), 3),
    ("sq_quant_weight_gateup", (_A, _A, 1, 48, 64, _A, _A, _A, None), 1),      # N_h not a multiple of 32
    ("sq_quant_weight_gateup", (_A, _U, 1, 64, 64, _A, _A, _A, None), 3),
    ("sq_smooth_quant_act", (_A, 1, 4, 64, _A, 2, _A, _A, None), 1),          # unknown mode
    ("sq_smooth_quant_act", (_A, 1, 4, 0, _A, 0, _A, _A, None), 1),
    ("sq_smooth_quant_act", (_A, 1, 4, 64, _A, 1, _A, _U, None), 3),
    ("sq_smooth_quant_act", (_A, 1, 0, 64, _A, 1, _A, _A, None), 0),          # no rows: nothing to do
    ("sq_rmsnorm_quant", (_A, 2, 4, 64, None, _A, 1e-5, _A, _A, None, None), 1),
    ("sq_rmsnorm_quant", (_A, 2, 4, 64, _A, _A, -1.0, _A, _A, None, None), 1),
    ("sq_rmsnorm_quant", (_A, 2, 4, 64, _A, _A, float("nan"), _A, _A, None, None), 1),
    ("sq_rmsnorm_quant", (_U, 2, 4, 64, _A, _A, 1e-5, _A, _A, None, None), 3),
    ("sq_rmsnorm_absmax", (_A, 2, 4, 0, _A, 1e-5, _A, None), 1),
    ("sq_rmsnorm_absmax", (_U, 2, 4, 64, _A, 1e-5, _A, None), 3),
    ("sq_rmsnorm_absmax", (_A, 2, 0, 64, _A, 1e-5, _A, None), 0),
    ("sq_linear_w8a8_gateup_silu", (_A, _A, 300, 96, 512, _A, 0, _A, _A, None, None, None, None), 1),   # N_h % 128
    ("sq_linear_w8a8_gateup_silu", (_A, _A, 300, 128, 512, _A, 0, _A, None, None, None, None, None), 1),  # no output
    ("sq_linear_w8a8_gateup_silu", (_A, _A, 300, 128, 512, _A, 0, _A, None, _A, None, _A, None), 1),   # hq without a2
    ("sq_linear_w8a8_gateup_silu", (_A, _A, 300, 128, 512, _A, 0, _A, _U, None, None, None, None), 3),
    ("sq_gemm_f16_ref", (_A, _A, 4, 40, 64, _A, None), 1),                    # N % 16
    ("sq_gemm_f16_ref", (_A, _A, 4, 32, 12, _A, None), 1),                    # K % 8
    ("sq_gemm_f16_ref", (_A, _A, 4, 32, 64, _U, None), 3),
    ("sq_sse_f16", (_A, _A, -1, _A, None), 1),
    ("sq_sse_f16", (_A, _U, 8, _A, None), 3),
    ("sq_sse_f16", (_A, _A, 0, _A, None), 0),
    ("sq_gemm_s32", (_A, _A, 4, 32, 64, None, None), 1),
    ("sq_gemm_s32", (_A, _A, 4, 32, 64, _U, None), 3),
    ("sq_linear_w8a8_noalloc", (_A, _A, 4, 32, 64, _A, 3, _A, None, 2, _A, None), 1),          # unknown mode
    ("sq_calib_absmax", (_A, 1, 0, 64, 64, _A, None), 0),
    ("sq_smooth_scales_fp8", (_A, _A, 64, 1.5, _A, None, None), 1),           # alpha outside [0, 1]
    ("sq_quant_weight_fp8", (_U, 1, 8, 64, _A, _A, _A, None), 3),
    ("sq_quant_weight_fp8", (_A, 7, 8, 64, _A, _A, _A, None), 1),               # unknown dtype
    ("sq_smooth_quant_act_fp8", (_A, 1, 4, 64, _A, 2, _A, _A, None), 1),        # unknown mode
    ("sq_smooth_quant_act_fp8", (_A, 1, 4, 64, _A, 1, _A, _U, None), 3),
    ("sq_linear_fp8", (_A, _A, 4, 40, 64, _A, 0, _A, None, 1, _A, None), 1),    # N % 16
    ("sq_linear_fp8", (_A, _A, 4, 32, 64, _A, 0, _A, None, 1, _U, None), 3),
    ("sq_linear_fp8", (_A, _A, 0, 32, 64, _A, 0, _A, None, 1, _A, None), 1),    # M = 0
    ("sq_calib_quantile", (_A, 1, 8, 64, 64, 0.0, _A, _A, 1 << 20, None), 1),   # p outside (0, 1]
    ("sq_calib_quantile", (_A, 1, 8, 64, 64, 0.5, _A, _A, 16, None), 6),        # workspace too small
    ("sq_calib_quantile", (_U, 1, 8, 64, 64, 0.5, _A, _A, 1 << 20, None), 3),
    ("sq_calib_quantile", (_A, 1, 8, 60, 60, 0.5, _A, _A, 1 << 20, None), 3),   # rows of 120 bytes
    ("sq_calib_batchmax_accumulate", (_A, 1, 0, 64, 64, _A, _A, None), 1),      # an empty batch
    ("sq_calib_mean_of_max", (_A, 64, 0, _A, None), 1),                          # no batches
    ("sq_quant_weight_fold", (_A, 1, 8, 64, _A, None, _A, _A, None), 1),         # s_next required
    ("sq_quant_weight_gateup_fold", (_A, _A, 1, 64, 64, _A, None, _A, _A, None), 1),
    ("sq_scales_to_f16", (_A, -1, _A, None), 1),
    ("sq_scales_from_f16", (None, 4, _A, None), 1),
    ("sq_linear_w8a8_f16scales", (_A, _A, 4, 40, 64, _A, 0, _A, None, 1, _A, None, 0, None), 1),   # N % 16
])
def test_every_entry_point_validates_before_launch(fn, args, status):
    import w8a8_post_quantization_calib_b200 as sq
    assert getattr(sq.lib(), fn)(*args) == status


def test_alpha_search_validation():
    import ctypes
    import w8a8_post_quantization_calib_b200 as sq
    lib = sq.lib()
    best = ctypes.c_float()
    # alphas must be ascending and within [0, 1]; 1..16 of them; a workspace is required
    assert lib.sq_alpha_search(_A, _A, 512, 256, 512, _A, _A, _alphas(0.5, 0.25), 2, _A, 1 << 30,
                               ctypes.byref(best), None, None) == 1
    assert lib.sq_alpha_search(_A, _A, 512, 256, 512, _A, _A, _alphas(0.5, 1.5), 2, _A, 1 << 30,
                               ctypes.byref(best), None, None) == 1
    assert lib.sq_alpha_search(_A, _A, 512, 256, 512, _A, _A, _alphas(0.5), 0, _A, 1 << 30,
                               ctypes.byref(best), None, None) == 1
    assert lib.sq_alpha_search(_A, _A, 512, 256, 512, _A, _A, _alphas(0.5), 1, None, 1 << 30,
                               ctypes.byref(best), None, None) == 1
    assert lib.sq_alpha_search(_A, _A, 512, 256, 512, _A, _A, _alphas(0.25, 0.5), 2, _A, 16,
                               ctypes.byref(best), None, None) == 6          # workspace too small



def test_noalloc_refuses_oversize_before_launch():
    """With the cluster split off (hook 2) the decode-size shape shares tiles
    through the fixed array; hook 4 makes the size check assume a 64 KiB
    array, which that schedule's partial sums do not fit."""
    import w8a8_post_quantization_calib_b200 as sq
    lib = sq.lib()
    lib.sq_debug_inject(2 | 4)
    try:
        assert lib.sq_linear_w8a8_noalloc(_A, _A, 16, 4096, 11008, _A, 1, _A, None, 2, _A, None) == 2
    finally:
        lib.sq_debug_inject(0)
