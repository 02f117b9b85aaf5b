"""Iterative refinement of the residual (test infrastructure; see the package header).

SVDQuant review (jeonghoonpark.com), §4.2, the list after the low-rank
decomposition equation: the low-rank decomposition is not done only once; R is
optimized repeatedly so that the quantization error is minimized.  The page
gives no algorithm.  Reading taken here: alternating minimization of the
weight-side error of the decomposition,

    E(L1 L2, R) = || W_hat - L1 L2 - Q(R) ||_F,      R = W_hat - L1 L2,

  step 0:  L1 L2 = SVD_r(W_hat)                    (plain SVDQuant, no refinement);
  step k:  L1 L2 = SVD_r(W_hat - Q(R_{k-1}))       (the best rank-r fit of what the
                                                    4-bit residual misses: with Q fixed,
                                                    Eckart-Young makes this exact),
           R_k   = W_hat - L1 L2                   (then quantized again).

Q is this oracle's NVFP4 weight quantizer (R rounded to float32, groups of 16
along K for every output column, per-tensor scale from R's own amax).  Because
the scales follow R, E need not fall at every step: the iterate with the
smallest E is kept (step 0 included, so refinement never does worse than one
decomposition).

Pins (tests/test_oracle_refine.py): zero steps reproduce the plain split;
every step's L1 L2 is the rank-r projection of W_hat - Q(R_{k-1}) computed by an
independent eigendecomposition; the kept error is the smallest of the history
and not above step 0's; r = 0 is a no-op; on outlier-channel data the error
falls.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List

import numpy as np

from .codec import dequantize
from .linear import pack_weight


def quantized_residual(R) -> np.ndarray:
    """Q(R) as a K x N float64 matrix: the NVFP4 weight quantizer applied to float32 R, dequantized."""
    pw = pack_weight(np.asarray(R, dtype=np.float64).astype(np.float32))
    return dequantize(pw.codes, pw.scales, pw.gs_w).T


def weight_error(W_hat, L1, L2, R) -> float:
    """|| W_hat - L1 L2 - Q(R) ||_F."""
    return float(np.linalg.norm(np.asarray(W_hat, dtype=np.float64) - L1 @ L2 - quantized_residual(R)))


@dataclass
class Step:
    L1: np.ndarray          # K x r
    L2: np.ndarray          # r x N
    R: np.ndarray           # K x N float64
    error: float            # || W_hat - L1 L2 - Q(R) ||_F
    target: np.ndarray      # the matrix whose rank-r SVD gave L1 L2 (W_hat at step 0)


def _rank_r(T, r: int):
    U, S, Vt = np.linalg.svd(T, full_matrices=False)
    return U[:, :r] * S[:r][None, :], Vt[:r, :]


def refine(W_hat, r: int, iters: int):
    """Returns (L1, L2, R, history): the kept decomposition and every step (step 0 first)."""
    W_hat = np.asarray(W_hat, dtype=np.float64)
    history: List[Step] = []
    target = W_hat
    for k in range(iters + 1):
        L1, L2 = _rank_r(target, r)
        R = W_hat - L1 @ L2
        QR = quantized_residual(R)
        history.append(Step(L1=L1, L2=L2, R=R, error=float(np.linalg.norm(W_hat - L1 @ L2 - QR)), target=target))
        target = W_hat - QR
    best = min(range(len(history)), key=lambda i: history[i].error)
    h = history[best]
    return h.L1, h.L2, h.R, history
