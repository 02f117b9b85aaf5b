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

Refinement (refine_iters > 0; SVDQuant review §4.2: R is optimized repeatedly
to minimize the quantization error, the page gives no algorithm): alternate
  L1 L2 = best rank-r fit of W_hat - Q(R_prev)   (truncated SVD; step 0 fits W_hat itself),
  R     = W_hat - L1 L2,
keeping the step with the smallest ||W_hat - L1 L2 - Q(R)||_F.  Q(R) is the
library's own quantizer: R is packed by svdq_pack_weight and read back with
svdq_dequant_weight on the GPU, so the residual is refined against exactly the
codes the layer will use.
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


def _rank_r(T: torch.Tensor, r: int):
    U, S, Vh = torch.linalg.svd(T, full_matrices=False)
    return U[:, :r] * S[:r][None, :], Vh[:r, :]


def quantize_residual_gpu(R: torch.Tensor, device) -> torch.Tensor:
    """Q(R) (K x N, float64 on the host) through the library's packing and dequantization kernels."""
    from . import svdq as C
    K, N = R.shape
    with torch.cuda.device(device):
        Rd = R.to(device, torch.float32).contiguous()
        Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
        SFw = torch.empty(C.svdq_sf_bytes(N, K), dtype=torch.uint8, device=device)
        gs = torch.empty(1, dtype=torch.float32, device=device)
        C.svdq_pack_weight(Rd, None, K, N, 0, Wq, SFw, gs, None)
        Rq = torch.empty((K, N), dtype=torch.float32, device=device)
        C.svdq_dequant_weight(Wq, SFw, gs, K, N, Rq)
        return Rq.to("cpu", torch.float64)


def refine_split(W_hat: torch.Tensor, r: int, iters: int, device):
    """Alternating refinement of the rank-r split against the 4-bit residual (see the module header).
    Returns (L1, L2, R, errors of every step)."""
    target = W_hat
    best, errors = None, []
    for _ in range(iters + 1):
        L1, L2 = _rank_r(target, r)
        R = W_hat - L1 @ L2
        QR = quantize_residual_gpu(R, device)
        err = float(torch.linalg.norm(W_hat - L1 @ L2 - QR))
        errors.append(err)
        if best is None or err < best[0]:
            best = (err, L1, L2, R)
        target = W_hat - QR
    return best[1], best[2], best[3], errors


def calibrate(X, W, r: int, alpha: float = 0.5, bias=None, lora_A=None, lora_B=None,
              X_cal=None, refine_iters: int = 0, device=None) -> LayerData:
    """Decompose W (K x N) for activations X (M x K); X_cal overrides the calibration activations.
    refine_iters > 0 refines the split against the 4-bit residual, quantized on `device` (a CUDA device)."""
    Wd = _as64(W)
    Xc = _as64(X if X_cal is None else X_cal)
    K, N = Wd.shape
    ax = Xc.abs().amax(dim=0)
    aw = Wd.abs().amax(dim=1)
    s = ax.pow(alpha) / aw.pow(1.0 - alpha)
    s = torch.where((ax == 0) | (aw == 0), torch.ones_like(s), s)
    W_hat = s[:, None] * Wd
    if refine_iters > 0:
        if device is None:
            raise ValueError("refinement quantizes the residual with the CUDA library: give a device")
        L1, L2, R, _ = refine_split(W_hat, r, refine_iters, torch.device(device))
    else:
        L1, L2 = _rank_r(W_hat, r)
        R = W_hat - L1 @ L2
    if lora_A is not None:
        L1 = torch.cat([L1, s[:, None] * _as64(lora_A)], dim=1)
        L2 = torch.cat([L2, _as64(lora_B)], dim=0)
    inv_s = (1.0 / s).to(torch.float32)
    L1fT = (L1 / s[:, None]).t().contiguous().to(torch.bfloat16)
    return LayerData(K=K, N=N, r=L1.shape[1], inv_s=inv_s, gs_x=act_global_scale(Xc, inv_s),
                     L1fT=L1fT, L2b=L2.contiguous().to(torch.bfloat16), R=R.to(torch.float32).contiguous(),
                     bias=None if bias is None else _as64(bias).to(torch.bfloat16), s=s)
