"""Shared test plumbing: host<->device copies of seeded inputs and bit comparisons."""
import numpy as np
import torch

import synth

F32, F16, BF16 = synth.F32, synth.F16, synth.BF16
TORCH_DT = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def dev(a: np.ndarray, dt: int | None = None) -> torch.Tensor:
    """numpy -> CUDA tensor.  uint16 arrays are 16-bit bit patterns of `dt`."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16).copy()).view(TORCH_DT[dt])
    else:
        t = torch.from_numpy(a.copy())
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy; 16-bit floats come back as uint16 bit patterns."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def bits_equal(a: np.ndarray, b: np.ndarray) -> bool:
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    if a.shape != b.shape:
        return False
    if a.dtype == np.float32:
        a = a.view(np.uint32)
    if b.dtype == np.float32:
        b = b.view(np.uint32)
    return np.array_equal(a, b)


def mismatch_report(a: np.ndarray, b: np.ndarray, n: int = 5) -> str:
    a = np.asarray(a)
    b = np.asarray(b)
    idx = np.argwhere(a != b)
    return f"{len(idx)} mismatches; first {idx[:n].tolist()}: got {a[tuple(idx[:n].T)]} want {b[tuple(idx[:n].T)]}"


def rel_err(a, b) -> np.ndarray:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.abs(a - b) / np.maximum(np.abs(b), 1e-300)


def rand_x(seed: int, shape, dt: int, sigma: float = 1.0, outliers: int = 0) -> np.ndarray:
    g = np.random.default_rng(seed)
    x = g.standard_normal(shape).astype(np.float32) * np.float32(sigma)
    if outliers:
        idx = g.choice(shape[1], size=outliers, replace=False)
        x[:, idx] *= g.uniform(20, 100, outliers).astype(np.float32)[None, :]
    return synth.cast(x, dt)
