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


# ------------------------------------------------------------------ on the GPU --
def randomized_rank_r(W_hat: torch.Tensor, r: int, oversample: int = 32, power_iters: int = 6,
                      seed: int = 0):
    """Rank-r factors (L1 = U_r Sigma_r, L2 = V_r^T) of a float64 K x N matrix on its device by a
    randomized range finder: Y = W_hat Omega (Omega Gaussian N x (r + oversample)), power_iters
    rounds of Y = W_hat (W_hat^T Q) with re-orthonormalization, then the exact SVD of the small
    B = Q^T W_hat.  The products are library float64 GEMMs and the orthonormalizations library QR
    factorizations (offline, outside the layer's forward pass)."""
    K, N = W_hat.shape
    ell = min(r + oversample, K, N)
    g = torch.Generator(device=W_hat.device).manual_seed(seed)
    Omega = torch.randn((N, ell), dtype=torch.float64, device=W_hat.device, generator=g)
    Q, _ = torch.linalg.qr(W_hat @ Omega)
    for _ in range(power_iters):
        Z, _ = torch.linalg.qr(W_hat.T @ Q)
        Q, _ = torch.linalg.qr(W_hat @ Z)
    B = Q.T @ W_hat
    Ub, S, Vh = torch.linalg.svd(B, full_matrices=False)
    U = Q @ Ub
    return U[:, :r] * S[:r][None, :], Vh[:r, :]


def calibrate_gpu(X, W, r: int, alpha: float = 0.5, bias=None, lora_A=None, lora_B=None, X_cal=None,
                  device=None, oversample: int = 32, power_iters: int = 6, seed: int = 0,
                  batch_rows: int = 8192) -> LayerData:
    """calibrate() with its statistics and its split on the GPU.

    Activation channel maxima stream over the calibration rows in batches (svdq_calib_absmax_cols,
    merged by max), weight channel maxima, smoothing factors and W_hat = diag(s) W come from the
    library's calibration kernels (float64 for everything weight-side), the rank-r split from
    randomized_rank_r, and gs_x from the maximum of f32(X * inv_s) (svdq_calib_act_amax).  The
    maxima, s and W_hat are those of calibrate(); the split differs from the exact truncated SVD only
    by the randomized range finder's approximation."""
    from . import svdq as C
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    Xc = X if X_cal is None else X_cal
    Xc = Xc if isinstance(Xc, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(Xc, dtype=np.float32))
    Wd = _as64(W)
    K, N = Wd.shape
    with torch.cuda.device(dev):
        Xb = Xc.to(torch.bfloat16)
        amax_x = torch.empty(K, dtype=torch.float32, device=dev)
        M = Xb.shape[0]
        for i, lo in enumerate(range(0, max(M, 1), batch_rows)):
            xb = Xb[lo:lo + batch_rows].to(dev).contiguous()
            C.svdq_calib_absmax_cols(xb, xb.shape[0], K, amax_x, accumulate=i > 0)
        W_dev = Wd.to(dev).contiguous()
        amax_w = torch.empty(K, dtype=torch.float64, device=dev)
        C.svdq_calib_absmax_rows(W_dev, K, N, amax_w)
        s = torch.empty(K, dtype=torch.float64, device=dev)
        inv_s = torch.empty(K, dtype=torch.float32, device=dev)
        C.svdq_calib_smooth(amax_x, amax_w, K, alpha, s, inv_s)
        W_hat = torch.empty_like(W_dev)
        C.svdq_calib_scale_rows(W_dev, s, K, N, W_hat)
        del W_dev
        L1, L2 = randomized_rank_r(W_hat, r, oversample, power_iters, seed)
        R = torch.addmm(W_hat, L1, L2, alpha=-1.0)
        del W_hat
        if lora_A is not None:
            L1 = torch.cat([L1, s[:, None] * _as64(lora_A).to(dev)], dim=1)
            L2 = torch.cat([L2, _as64(lora_B).to(dev)], dim=0)
        amax = torch.empty(1, dtype=torch.float32, device=dev)
        for i, lo in enumerate(range(0, max(M, 1), batch_rows)):
            xb = Xb[lo:lo + batch_rows].to(dev).contiguous()
            C.svdq_calib_act_amax(xb, xb.shape[0], K, inv_s, amax, accumulate=i > 0)
        a = float(amax.item())
        gs_x = 1.0 if a == 0.0 else float(np.float32(np.float64(a) / 2688.0))
        L1fT = (L1 / s[:, None]).t().contiguous().to(torch.bfloat16)
        return LayerData(K=K, N=N, r=L1.shape[1], inv_s=inv_s.cpu(), gs_x=gs_x, L1fT=L1fT.cpu(),
                         L2b=L2.contiguous().to(torch.bfloat16).cpu(), R=R.to(torch.float32).contiguous().cpu(),
                         bias=None if bias is None else _as64(bias).to(torch.bfloat16), s=s.cpu())
