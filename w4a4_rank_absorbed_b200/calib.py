"""Offline calibration and decomposition of one SVDQuant layer (float64, host side).

Computed once per layer and handed to the CUDA kernels as data ("From
SmoothQuant to SVDQuant", section quantization scheme: the weight-side
scales, the smoothing factors and the low-rank branch are fixed offline).

  s_j   = max|X_j|^alpha / max|W_j|^(1-alpha)       (Smooth Quant (W8A8) section; s_j = 1 if a max is 0)
  W_hat = diag(s) W;  W_hat = U Sigma V^T;  L1 = U_r Sigma_r,  L2 = V_r^T,  R = W_hat - L1 L2
                                                     (SVDQuant review §4.2; rank 32 by default)
  LoRA  : L1 <- [L1 | diag(s) A],  L2 <- [L2 ; B]   (adapters join the low-rank branch, R unchanged)
  data  : inv_s = f32(1/s), L1f^T = bf16(diag(s)^-1 L1)^T (r x K), L2b = bf16(L2) (r x N),
          R float32 (K x N), gs_x = f32(amax(f32(X * inv_s)) / 2688) from the calibration activations.

Uses torch CPU float64 linear algebra.  This is preparation of the layer's
constants, not a step of the forward pass.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch


@dataclass
class LayerData:
    K: int
    N: int
    r: int
    inv_s: torch.Tensor     # float32 [K]
    gs_x: float             # static activation global scale (float32 value)
    L1fT: torch.Tensor      # bf16 [r, K]
    L2b: torch.Tensor       # bf16 [r, N]
    R: torch.Tensor         # float32 [K, N]
    bias: Optional[torch.Tensor]  # bf16 [N]
    s: torch.Tensor         # float64 [K]


def _as64(a) -> torch.Tensor:
    if isinstance(a, torch.Tensor):
        return a.detach().to("cpu", torch.float64)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def act_global_scale(X, inv_s: torch.Tensor) -> float:
    """f32(amax(f32(X * inv_s)) / 2688), or 1.0 when the activations are all zero."""
    xh = _as64(X).to(torch.float32) * inv_s.to(torch.float32)
    amax = xh.abs().max() if xh.numel() else torch.tensor(0.0, dtype=torch.float32)
    if float(amax) == 0.0:
        return 1.0
    return float(amax / torch.tensor(2688.0, dtype=torch.float32))


def calibrate(X, W, r: int, alpha: float = 0.5, bias=None, lora_A=None, lora_B=None,
              X_cal=None) -> LayerData:
    """Decompose W (K x N) for activations X (M x K); X_cal overrides the calibration activations."""
    Wd = _as64(W)
    Xc = _as64(X if X_cal is None else X_cal)
    K, N = Wd.shape
    ax = Xc.abs().amax(dim=0)
    aw = Wd.abs().amax(dim=1)
    s = ax.pow(alpha) / aw.pow(1.0 - alpha)
    s = torch.where((ax == 0) | (aw == 0), torch.ones_like(s), s)
    W_hat = s[:, None] * Wd
    U, S, Vh = torch.linalg.svd(W_hat, full_matrices=False)
    L1 = U[:, :r] * S[:r][None, :]
    L2 = Vh[:r, :]
    R = W_hat - L1 @ L2
    if lora_A is not None:
        L1 = torch.cat([L1, s[:, None] * _as64(lora_A)], dim=1)
        L2 = torch.cat([L2, _as64(lora_B)], dim=0)
    inv_s = (1.0 / s).to(torch.float32)
    L1fT = (L1 / s[:, None]).t().contiguous().to(torch.bfloat16)
    return LayerData(K=K, N=N, r=L1.shape[1], inv_s=inv_s, gs_x=act_global_scale(Xc, inv_s),
                     L1fT=L1fT, L2b=L2.contiguous().to(torch.bfloat16), R=R.to(torch.float32).contiguous(),
                     bias=None if bias is None else _as64(bias).to(torch.bfloat16), s=s)
