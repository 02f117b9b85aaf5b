"""Offline decomposition of the oracle (test infrastructure; see the package header).

Computed once per layer in float64 (the pages keep these quantities static:
"From SmoothQuant to SVDQuant", section quantization scheme, item 1 -- the
weight scales, the smoothing factors and the low-rank branch are fixed at
calibration and written into the model).

  * Smoothing ("From SmoothQuant to SVDQuant", section Smooth Quant (W8A8)):
        Y = (X diag(s)^-1) (diag(s) W) = X_hat W_hat,
        s_j = max|X_j|^alpha / max|W_j|^(1 - alpha),
    X_j the j-th input channel (column of X), W_j the j-th row of W (K x N).
    Reading: s_j = 1 when either maximum is 0 (the pages are silent).
  * Low-rank branch (SVDQuant review, §4.2; "From SmoothQuant to SVDQuant",
    section SVD decomposition / quantization scheme): W_hat = U Sigma V^T,
    keep the r largest singular values, L1 = U_r Sigma_r (K x r),
    L2 = V_r^T (r x N), residual R = W_hat - L1 L2; only R is quantized to 4 bits.
  * LoRA (abstract of "SVDQuant: Absorbing Outliers by Low-Rank Components
    for 4-Bit Diffusion Models": adapters join the low-rank branch with no
    re-quantization).  Reading: an adapter X A B is appended as
    L1 <- [L1 | diag(s) A], L2 <- [L2 ; B], so X_hat diag(s) A B = X A B and R is unchanged.
  * Data handed to the layer (reading: the pages keep the low-rank branch in
    16 bits; bf16 is taken): L1f = bf16(diag(s)^-1 L1) (smoothing folded in,
    one rounding from float64), L2b = bf16(L2), inv_s = f32(1 / s),
    R as float32, and the static activation scale gs_x = f32(amax(X_hat)/2688)
    with X_hat = f32(X * inv_s) from the calibration activations.

Pins (tests/test_oracle_decompose.py): the smoothing identity
X diag(s)^-1 diag(s) W = X W; W_hat = L1 L2 + R; Eckart-Young
(||R||_F^2 equals the sum of the discarded squared singular values,
||R||_2 = sigma_{r+1}); the rank-r product against an independent
eigendecomposition of W_hat^T W_hat.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .codec import global_scale

F32 = np.float32


def bf16_round(a) -> np.ndarray:
    """Round float64 to the nearest bfloat16 value, ties to even; float64 result (exact frexp/rint).

    bfloat16 keeps 8 significant bits down to its smallest normal 2^-126 and a fixed spacing of
    2^-133 below it (subnormals); magnitudes that round to 2^128 or beyond become infinite."""
    a = np.asarray(a, dtype=np.float64)
    _, e = np.frexp(a)                       # |a| = m 2^e, 0.5 <= m < 1
    q = np.maximum(e - 8, -133)              # exponent of the spacing at |a|
    r = np.ldexp(np.rint(np.ldexp(a, -q)), q)
    with np.errstate(invalid="ignore"):
        return np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, a), r)


def smoothing_factors(X, W, alpha: float) -> np.ndarray:
    amax_x = np.abs(np.asarray(X, dtype=np.float64)).max(axis=0)
    amax_w = np.abs(np.asarray(W, dtype=np.float64)).max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = amax_x ** alpha / amax_w ** (1.0 - alpha)
    s[(amax_x == 0) | (amax_w == 0)] = 1.0
    return s


def low_rank_split(W_hat, r: int):
    """Truncated SVD: (L1 = U_r Sigma_r, L2 = V_r^T, R = W_hat - L1 L2, all singular values)."""
    U, S, Vt = np.linalg.svd(np.asarray(W_hat, dtype=np.float64), full_matrices=False)
    L1 = U[:, :r] * S[:r][None, :]
    L2 = Vt[:r, :]
    R = W_hat - L1 @ L2
    return L1, L2, R, S


@dataclass
class Decomposition:
    s: np.ndarray          # K, float64
    inv_s: np.ndarray      # K, float32
    L1: np.ndarray         # K x r_eff float64 (smoothed space, LoRA appended)
    L2: np.ndarray         # r_eff x N float64
    R: np.ndarray          # K x N float64 residual
    R32: np.ndarray        # K x N float32 (what is quantized)
    L1f: np.ndarray        # K x r_eff, bf16 values as float64
    L2b: np.ndarray        # r_eff x N, bf16 values as float64
    gs_x: np.float32       # static activation global scale
    sigma: np.ndarray      # singular values of W_hat


def activation_global_scale(X, inv_s) -> np.float32:
    """gs_x from calibration activations: amax over X_hat = f32(X * inv_s)."""
    xh = (np.asarray(X, dtype=np.float32) * np.asarray(inv_s, dtype=np.float32)).astype(np.float32)
    return global_scale(np.abs(xh).max() if xh.size else 0.0)


def decompose(X, W, r: int, alpha: float = 0.5, lora_A: Optional[np.ndarray] = None,
              lora_B: Optional[np.ndarray] = None, X_cal=None, refine_iters: int = 0) -> Decomposition:
    """refine_iters > 0: the low-rank split is refined against the 4-bit residual (oracle.refine)."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    Xc = X if X_cal is None else np.asarray(X_cal, dtype=np.float64)
    s = smoothing_factors(Xc, W, alpha)
    W_hat = s[:, None] * W
    L1, L2, R, S = low_rank_split(W_hat, r)
    if refine_iters > 0:
        from .refine import refine
        L1, L2, R, _ = refine(W_hat, r, refine_iters)
    if lora_A is not None:
        L1 = np.concatenate([L1, s[:, None] * lora_A], axis=1)
        L2 = np.concatenate([L2, lora_B], axis=0)
    inv_s = (1.0 / s).astype(np.float32)
    L1f = bf16_round(L1 / s[:, None])
    L2b = bf16_round(L2)
    return Decomposition(s=s, inv_s=inv_s, L1=L1, L2=L2, R=R, R32=R.astype(np.float32),
                         L1f=L1f, L2b=L2b, gs_x=activation_global_scale(Xc, inv_s), sigma=S)
