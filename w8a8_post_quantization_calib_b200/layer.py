"""Layer-level driver of the SmoothQuant W8A8 linear on top of the C ABI.

Mirrors the calibration -> offline transform -> runtime flow of the
"010. SmoothQuant Integration" design (SmoothQuantQuantizer.add_batch keeps
the per-channel max-abs; the layer holds int8 weights with per-row scales,
the per-channel smoothing factors and the activation scale).  PyTorch only
allocates device buffers; every computation is a libsq call.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (ACT_PER_TOKEN, ACT_STATIC, calib_absmax, linear_w8a8, linear_workspace_size, quant_weight,
               smooth_quant_act, smooth_scales)


class Calibrator:
    """Running per-channel max|X_j| over calibration batches (one layer)."""

    def __init__(self, K: int, device="cuda"):
        self.act_max = torch.zeros(K, dtype=torch.float32, device=device)

    def add_batch(self, x: torch.Tensor, stream=None) -> None:
        calib_absmax(x.reshape(-1, x.shape[-1]), self.act_max, stream=stream)


@dataclass
class QuantizedLinear:
    wq: torch.Tensor          # int8 [N, K]
    w_scale: torch.Tensor     # fp32 [N]
    s: torch.Tensor           # fp32 [K]
    a_static: torch.Tensor    # fp32 [1]
    act_max: torch.Tensor     # fp32 [K]
    w_max: torch.Tensor       # fp32 [K]
    alpha: float
    mode: int = ACT_STATIC
    bias: torch.Tensor | None = None

    @property
    def N(self) -> int:
        return self.wq.shape[0]

    @property
    def K(self) -> int:
        return self.wq.shape[1]

    @classmethod
    def from_float(cls, w: torch.Tensor, act_max: torch.Tensor, alpha: float = 0.5, mode: int = ACT_STATIC,
                   bias=None, stream=None) -> "QuantizedLinear":
        N, K = w.shape
        dev = w.device
        w_max = torch.zeros(K, dtype=torch.float32, device=dev)
        calib_absmax(w, w_max, stream=stream)
        s = torch.empty(K, dtype=torch.float32, device=dev)
        a = torch.empty(1, dtype=torch.float32, device=dev)
        smooth_scales(act_max, w_max, alpha, s, a, stream=stream)
        wq = torch.empty(N, K, dtype=torch.int8, device=dev)
        ws = torch.empty(N, dtype=torch.float32, device=dev)
        quant_weight(w, s, wq, ws, stream=stream)
        return cls(wq, ws, s, a, act_max, w_max, alpha, mode, bias)

    def quantize_input(self, x: torch.Tensor, xq=None, a_scale=None, stream=None):
        M = x.shape[0]
        if xq is None:
            xq = torch.empty(M, self.K, dtype=torch.int8, device=x.device)
        if self.mode == ACT_STATIC:
            a_scale = self.a_static
        elif a_scale is None:
            a_scale = torch.empty(M, dtype=torch.float32, device=x.device)
        smooth_quant_act(x, self.s, self.mode, a_scale, xq, stream=stream)
        return xq, a_scale

    def workspace(self, M: int, device="cuda") -> torch.Tensor | None:
        n = linear_workspace_size(M, self.N, self.K)
        return torch.zeros(n, dtype=torch.uint8, device=device) if n else None

    def forward(self, x: torch.Tensor, out_dtype=torch.float16, y=None, workspace=None, stream=None):
        M = x.shape[0]
        xq, a = self.quantize_input(x, stream=stream)
        if y is None:
            y = torch.empty(M, self.N, dtype=out_dtype, device=x.device)
        linear_w8a8(xq, self.wq, a, self.mode, self.w_scale, y, bias=self.bias, workspace=workspace,
                    stream=stream)
        return y


__all__ = ["Calibrator", "QuantizedLinear", "ACT_STATIC", "ACT_PER_TOKEN"]
