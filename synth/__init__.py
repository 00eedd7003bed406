"""Seeded synthetic inputs for the SmoothQuant W8A8 linear layer.

This module only draws random numbers and casts them to storage dtypes: it
holds none of the method's arithmetic, so both the CUDA path's tests and the
CPU oracle can take their inputs from it.

Generators are numpy PCG64 with seed = 1000 * workload + stream.  Values are
drawn in fp32 and rounded (RNE) to the storage dtype: fp16 through numpy,
bf16 through torch's CPU cast.  16-bit tensors are returned as uint16 bit
patterns (bf16 has no numpy dtype); ``as_f16`` views fp16 bits as float16.

Activation laws (outlier channels are held at the same columns and the same
scale for every token, calibration and runtime alike: the pages describe
outliers as systematic, channel-bound features):
  * "linear toy": X ~ N(0, 5^2), channel 50 set to 100.0; W ~ N(0, 1)
    (the tbr8.org toy example's law, K=1024, N=2048)
  * "outlier": X ~ N(0,1), round(0.5% K) seeded channels scaled by
    c_j ~ U(20, 100); W ~ N(0, 0.02^2)
  * "heavy tail": X ~ Student-t(3), round(1% K) seeded channels x50
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F32, F16, BF16 = 0, 1, 2


def rng(workload: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * workload + stream))


def cast(a: np.ndarray, dt: int) -> np.ndarray:
    """fp32 -> storage dtype (RNE).  16-bit results are uint16 bit patterns."""
    a = np.ascontiguousarray(a, np.float32)
    if dt == F32:
        return a
    if dt == F16:
        return a.astype(np.float16).view(np.uint16)
    import torch
    t = torch.from_numpy(a).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def as_f16(bits: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(bits).view(np.float16)


def normal(g: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return x


def outlier_channels(g: np.random.Generator, K: int, frac: float, lo: float, hi: float | None):
    """Seeded outlier channel indices (without replacement) and their scales."""
    n = max(1, int(round(frac * K)))
    idx = np.sort(g.choice(K, size=n, replace=False))
    if hi is None:
        c = np.full(n, lo, np.float32)
    else:
        c = g.uniform(lo, hi, size=n).astype(np.float32)
    return idx, c


def apply_channels(x: np.ndarray, idx: np.ndarray, c: np.ndarray) -> np.ndarray:
    x[:, idx] *= c[None, :]
    return x


@dataclass
class LinearWorkload:
    """One linear layer: calibration batches, runtime batch, weight (+ bias)."""
    name: str
    K: int
    N: int
    M: int
    x_dt: int
    w_dt: int
    out_dt: int
    calib: list = field(default_factory=list)   # list of [rows, K] arrays (storage dtype)
    x: np.ndarray | None = None                 # [M, K] runtime batch
    w: np.ndarray | None = None                 # [N, K]
    alpha: float = 0.5
    mode: int = 0                               # 0 static, 1 per-token
    outlier_idx: np.ndarray | None = None


def linear_toy(M: int = 16, K: int = 1024, N: int = 2048, calib_batches: int = 4,
               workload: int = 1, outlier: bool = True) -> LinearWorkload:
    """Single linear, fp32: X ~ N(0, 5^2) with channel 50 = 100.0; W ~ N(0, 1)."""
    def act(stream, rows):
        x = normal(rng(workload, stream), (rows, K), 5.0)
        if outlier:
            x[:, 50] = 100.0
        return x
    wl = LinearWorkload("linear toy", K, N, M, F32, F32, F32)
    wl.calib = [act(10 + b, M) for b in range(calib_batches)]
    wl.x = act(2, M)
    wl.w = normal(rng(workload, 3), (N, K), 1.0)
    wl.outlier_idx = np.array([50]) if outlier else np.array([], np.int64)
    return wl


def outlier_linear(M: int, K: int, N: int, calib_batches: int, calib_rows: int,
                   x_dt: int, w_dt: int, out_dt: int, workload: int, mode: int = 0,
                   frac: float = 0.005, lo: float = 20.0, hi: float | None = 100.0,
                   heavy_tail: bool = False, w_sigma: float = 0.02, shard: int = 0) -> LinearWorkload:
    """Llama-shaped linear with seeded, token-consistent outlier channels.

    ``shard`` selects an independent set of calibration and runtime token
    batches (same layer, same weight, same outlier channels): one per rank
    when the token batches are spread over several GPUs.
    """
    idx, c = outlier_channels(rng(workload, 1), K, frac, lo, hi)

    def act(stream, rows):
        g = rng(workload, stream)
        if heavy_tail:
            x = g.standard_t(3, size=(rows, K)).astype(np.float32)
        else:
            x = normal(g, (rows, K))
        return cast(apply_channels(x, idx, c), x_dt)

    wl = LinearWorkload("outlier linear", K, N, M, x_dt, w_dt, out_dt, mode=mode)
    wl.calib = [act(100 + b + 100000 * shard, calib_rows) for b in range(calib_batches)]
    wl.x = act(2 + 100000 * shard, M)
    wl.w = cast(normal(rng(workload, 3), (N, K), w_sigma), w_dt)
    wl.outlier_idx = idx
    return wl


def qkv_7b(M: int = 2048, K: int = 4096, N: int = 12288, calib_batches: int = 64,
           calib_rows: int = 512, shard: int = 0) -> LinearWorkload:
    """Llama-7B-shaped QKV projection: fp16 X and W, static scale, fp16 out."""
    return outlier_linear(M, K, N, calib_batches, calib_rows, F16, F16, F16, workload=2, shard=shard)


def mlp_7b(which: str, M: int, calib_batches: int = 64, calib_rows: int = 512,
           K: int | None = None, N: int | None = None) -> LinearWorkload:
    """Llama-7B MLP pair ('up': 4096->11008, 'down': 11008->4096); per-token, bf16."""
    if which == "up":
        K = K or 4096
        N = N or 11008
        wl_id = 3
    else:
        K = K or 11008
        N = N or 4096
        wl_id = 30
    return outlier_linear(M, K, N, calib_batches, calib_rows, BF16, BF16, BF16,
                          workload=wl_id, mode=1)


def heavy_13b(M: int = 8192, K: int = 5120, N: int = 13824, calib_batches: int = 16,
              calib_rows: int = 512) -> LinearWorkload:
    """13B-shaped linear: Student-t(3) activations + 1% channels x50; fp16; alpha search."""
    return outlier_linear(M, K, N, calib_batches, calib_rows, F16, F16, F16, workload=4,
                          frac=0.01, lo=50.0, hi=None, heavy_tail=True)


@dataclass
class MLPBlockWorkload:
    """70B-shaped decoder MLP block (RMSNorm -> gate/up -> SiLU*mul -> down), bf16."""
    M: int
    d: int
    f: int
    x: np.ndarray
    calib: list
    gamma: np.ndarray
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    eps: float = 1e-5
    alpha: float = 0.5


def mlp_block_70b(M: int = 16384, d: int = 8192, f: int = 28672, calib_batches: int = 8,
                  calib_rows: int = 2048, gamma_random: bool = False, shard: int = 0) -> MLPBlockWorkload:
    """``shard`` selects independent calibration and runtime token batches (same
    block weights and outlier channels): one set per rank when the tokens are
    spread over several GPUs."""
    wl = 5
    idx, c = outlier_channels(rng(wl, 1), d, 0.005, 20.0, 100.0)

    def act(stream, rows):
        return cast(apply_channels(normal(rng(wl, stream + 100000 * shard), (rows, d)), idx, c), BF16)

    gamma = (rng(wl, 4).uniform(0.5, 1.5, size=d).astype(np.float32) if gamma_random
             else np.ones(d, np.float32))
    return MLPBlockWorkload(
        M=M, d=d, f=f, x=act(2, M), calib=[act(100 + b, calib_rows) for b in range(calib_batches)],
        gamma=gamma,
        w_gate=cast(normal(rng(wl, 5), (f, d), 0.02), BF16),
        w_up=cast(normal(rng(wl, 6), (f, d), 0.02), BF16),
        w_down=cast(normal(rng(wl, 7), (d, f), 0.02), BF16))
