"""Build libsq.so (the CUDA kernels + C ABI) and libsq_peak.so (the tensor-core
peak measurement used as the GEMM roofline denominator) in-tree with nvcc for
sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libsq.so")
SOURCES = ["libsq.cu"]
HEADERS = ["common.cuh", "ptx_sm100.cuh", "calib.cuh", "quant.cuh", "gemm.cuh"]
PEAK_SO = os.path.join(HERE, "libsq_peak.so")
PEAK_SOURCES = ["peak.cu"]
PEAK_HEADERS = ["common.cuh", "ptx_sm100.cuh"]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    return "nvcc"


def _stale(so: str, sources, headers) -> bool:
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    deps = [os.path.join(CSRC, f) for f in list(sources) + list(headers)] + [os.path.join(ROOT, "include", "sq.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(so: str, sources, verbose: bool, extra) -> None:
    tmp = so + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(extra or []), "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", tmp, *[os.path.join(CSRC, f) for f in sources]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, so)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if force or _stale(SO, SOURCES, HEADERS):
        _compile(SO, SOURCES, verbose, extra)
    if force or _stale(PEAK_SO, PEAK_SOURCES, PEAK_HEADERS):
        _compile(PEAK_SO, PEAK_SOURCES, verbose, extra)
    return SO


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
