"""The SVDQuant linear layer in the oracle (test infrastructure; see the package header).

Output (SVDQuant review, §4.2, the low-rank decomposition equation):
    X W = X_hat W_hat = X_hat L1 L2 + X_hat R
        ~ X_hat L1 L2 (16-bit low-rank branch) + Q(X_hat) Q(R) (4-bit residual),
plus the layer bias.  With the smoothing folded into the stored down factor
(L1f = diag(s)^-1 L1, see ``decompose``), the low-rank branch is X L1f L2b.
The 4-bit branch is the scaled product of §3 (XW ~ s_X s_W Q_X Q_W) in its
block-scaled form: sum over K of code_x * sb_x * code_w * sb_w, times
gs_x * gs_w.

The three functions below split the layer the way the library does
(weight packing, activation quantization with the down-projection, the
4-bit GEMM with the up-projection); ``svdq_reference`` chains them.
Everything after the quantizer's decisions is float64 from dequantized
values: no blocking, fusion or reordering.

Pins (tests/test_oracle_linear.py): a pure-Python triple loop on tiny
inputs; the blocked form sum_g s_g (Q_X,g . Q_W,g) equals the dequantized
product; the error bound of §4.1 (the four factors); the method effect
(SVDQuant error below plain W4A4 error on outlier-channel data).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .codec import dequantize, global_scale, nvfp4_quantize, pack_codes
from .layout import sf_to_storage

F32 = np.float32


@dataclass
class PackedWeight:
    codes: np.ndarray      # N x K, one E2M1 code per byte
    scales: np.ndarray     # N x K/16 UE4M3
    gs_w: np.float32


@dataclass
class QuantAct:
    codes: np.ndarray      # M x K
    scales: np.ndarray     # M x K/16
    LA: np.ndarray         # M x r float64: X L1f (= X_hat L1 up to the bf16 rounding of L1f)


def pack_weight(R32) -> PackedWeight:
    """Static weight quantization of the residual R (K x N, float32): groups of 16 along K per column n."""
    R32 = np.asarray(R32, dtype=np.float32)
    gs_w = global_scale(np.abs(R32).max() if R32.size else 0.0)
    codes, scales = nvfp4_quantize(np.ascontiguousarray(R32.T), gs_w)
    return PackedWeight(codes=codes, scales=scales, gs_w=gs_w)


def quantize_act(X, inv_s, gs_x, L1f: Optional[np.ndarray]) -> QuantAct:
    """X_hat = f32(X * inv_s) (the smoothing divide), NVFP4 codes of X_hat, and X L1f in float64."""
    X = np.asarray(X, dtype=np.float64)
    xh = (X.astype(np.float32) * np.asarray(inv_s, dtype=np.float32)).astype(np.float32)
    codes, scales = nvfp4_quantize(xh, gs_x)
    LA = X @ np.asarray(L1f, dtype=np.float64) if L1f is not None and L1f.shape[1] else np.zeros((X.shape[0], 0))
    return QuantAct(codes=codes, scales=scales, LA=LA)


def linear(qa: QuantAct, gs_x, pw: PackedWeight, L2b: Optional[np.ndarray], bias: Optional[np.ndarray]) -> np.ndarray:
    """Y = gs_x gs_w sum_k dec(x) dec(w) + LA L2b + bias, float64."""
    Xd = dequantize(qa.codes, qa.scales, gs_x)
    Wd = dequantize(pw.codes, pw.scales, pw.gs_w)
    Y = Xd @ Wd.T
    if L2b is not None and L2b.shape[0]:
        Y = Y + qa.LA @ np.asarray(L2b, dtype=np.float64)
    if bias is not None:
        Y = Y + np.asarray(bias, dtype=np.float64)[None, :]
    return Y


def svdq_reference(X, inv_s, gs_x, L1f, L2b, R32, bias):
    """The whole layer: returns (Y float64, QuantAct, PackedWeight)."""
    pw = pack_weight(R32)
    qa = quantize_act(X, inv_s, gs_x, L1f)
    return linear(qa, gs_x, pw, L2b, bias), qa, pw


def storage_views(qa: QuantAct, pw: PackedWeight):
    """Byte buffers in the library's storage formats (packed codes, scale order), for comparisons."""
    return {
        "Xq": pack_codes(qa.codes), "SFx": sf_to_storage(qa.scales),
        "Wq": pack_codes(pw.codes), "SFw": sf_to_storage(pw.scales),
    }


# ------------------------------------------------------------ baselines ------
def fake_quant(T32, gs=None):
    """Dequantized NVFP4 image of a float32 matrix quantized along its rows' K axis."""
    T32 = np.asarray(T32, dtype=np.float32)
    if gs is None:
        gs = global_scale(np.abs(T32).max() if T32.size else 0.0)
    codes, scales = nvfp4_quantize(T32, gs)
    return dequantize(codes, scales, gs)


def w4a4_plain(X, W, bias):
    """Plain NVFP4 W4A4: no smoothing, no low-rank branch (baseline of §3)."""
    Xd = fake_quant(np.asarray(X, dtype=np.float32))
    Wd = fake_quant(np.ascontiguousarray(np.asarray(W, dtype=np.float32).T))
    return Xd @ Wd.T + np.asarray(bias)[None, :]


def w4a4_smooth_only(X, W, s, bias):
    """Smoothing then NVFP4 W4A4 of X_hat and W_hat, no low-rank branch (§4.2, 'after smoothing')."""
    xh = (np.asarray(X, dtype=np.float64) / s[None, :]).astype(np.float32)
    wh = (s[:, None] * np.asarray(W, dtype=np.float64)).astype(np.float32)
    Xd = fake_quant(xh)
    Wd = fake_quant(np.ascontiguousarray(wh.T))
    return Xd @ Wd.T + np.asarray(bias)[None, :]


def rel_fro(A, B) -> float:
    """||A - B||_F / ||B||_F."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    return float(np.linalg.norm(A - B) / max(np.linalg.norm(B), 1e-300))
