"""Measured dense tensor-core peak of the current GPU (INT8 kind::i8 and FP8
kind::f8f6f4), the denominator of the GEMMs' roofline fractions.

``libsq_peak.so`` runs the GEMM's tcgen05 mainloop on shared-memory-resident
operands (no operand traffic, no epilogue) on every SM pair; this module times
its launches with CUDA events on the current stream.  ``burst`` is one launch
of about ``ms`` milliseconds after a warm-up launch (the rate a kernel timed
alone sees); ``sustained`` is back-to-back launches for about ``seconds``
(the rate a kernel inside a long step sees under the power cap).

``stream_read`` launches the library's streaming read of one buffer: the
ceiling of a kernel that reads the same bytes once per launch (a decode-size
GEMM's weights), against which the bench reports the small-M GEMMs.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsq_peak.so")
KINDS = {"i8": 0, "e4m3": 2}
MACS_PER_ITER = 256 * 256 * 128          # one 128-byte K block of a 256 x 256 pair tile
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m w8a8_post_quantization_calib_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.sqpeak_clusters.restype = ctypes.c_int
        L.sqpeak_clusters.argtypes = [ctypes.c_int]
        L.sqpeak_launch.restype = ctypes.c_int
        L.sqpeak_launch.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        L.sqpeak_error_word.restype = ctypes.c_int
        L.sqpeak_error_word.argtypes = []
        L.sqpeak_stream_read.restype = ctypes.c_int
        L.sqpeak_stream_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_void_p]
        _lib = L
    return _lib


def _launch(kind: int, clusters: int, iters: int) -> None:
    st = torch.cuda.current_stream().cuda_stream
    rc = lib().sqpeak_launch(kind, clusters, iters, st)
    if rc != 0:
        raise RuntimeError(f"sqpeak_launch: cudaError {rc}")


def _timed(kind: int, clusters: int, iters: int, launches: int) -> float:
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(launches):
        _launch(kind, clusters, iters)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def measure(kind: str = "i8", ms: float = 100.0, seconds: float = 0.0) -> dict:
    """Returns {"tops", "ms", "launches", "iters", "clusters"} for one burst
    launch of ~ms (seconds == 0) or back-to-back launches for ~seconds."""
    k = KINDS[kind]
    clusters = lib().sqpeak_clusters(k)
    if clusters <= 0:
        raise RuntimeError("sqpeak_clusters failed")
    # size one launch to ~ms from a short probe
    it0 = 2000
    _timed(k, clusters, it0, 1)
    t0 = _timed(k, clusters, it0, 1)
    iters = min(1 << 20, max(it0, int(it0 * ms / max(t0, 1e-3))))
    _timed(k, clusters, iters, 1)                       # warm-up at the measured size
    launches = max(1, int(round(seconds * 1e3 / ms))) if seconds > 0 else 1
    t = _timed(k, clusters, iters, launches)
    if lib().sqpeak_error_word() != 0:
        raise RuntimeError("peak kernel: a bounded wait timed out")
    ops = 2.0 * MACS_PER_ITER * iters * clusters * launches
    return {"tops": ops / (t * 1e-3) / 1e12, "ms": t, "launches": launches, "iters": iters, "clusters": clusters}


def stream_read(buf: torch.Tensor, blocks: int, sink: torch.Tensor) -> None:
    """One launch reading every byte of the contiguous CUDA tensor `buf` once
    (the ceiling of a kernel that streams it once) on the current stream."""
    rc = lib().sqpeak_stream_read(buf.data_ptr(), buf.numel() * buf.element_size(), int(blocks), sink.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"sqpeak_stream_read: cudaError {rc}")
