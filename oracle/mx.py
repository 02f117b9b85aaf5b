"""MXFP4 codec and layer of the oracle (test infrastructure; see the package header).

The pages name MXFP4 as one of the 4-bit formats the method is applied to next
to NVFP4 (the WUSH summary page: format compatibility and the MXFP4 / NVFP4 /
INT4 evaluations; "From SmoothQuant to SVDQuant", personal view, contrasts
NVFP4's group of 16 with coarser groups) but do not define it.  Reading taken
here: the Microscaling (MX) FP4 format as its public specification defines it.

  * blocks of 32 consecutive values along K (both operands, as block-scaled
    MMA requires);
  * elements FP4 E2M1 (the same grid as NVFP4: 0, 0.5, 1, 1.5, 2, 3, 4, 6);
  * one shared scale per block, an E8M0 byte e standing for 2^(e - 127)
    (e = 255 is NaN and is never produced);
  * the scale exponent X = floor(log2(amax)) - 2, 2 being the exponent of the
    largest E2M1 normal (6 = 1.5 * 2^2), clamped to [-127, 127]; an all-zero
    block takes e = 0;
  * code = E2M1_rne_satfinite(x * 2^-X): the product is exact (a power of
    two), the one rounding is the E2M1 one; values from 6 up to 8 saturate
    to 6, which is the format's own clipping;
  * no per-tensor scale.

The MX layer is the SVDQuant layer of oracle.linear with this codec in place
of NVFP4: Y = sum_k dec(x) dec(w) + (X L1f) L2b + bias (global scales 1).

Pins (tests/test_oracle_mx.py): E8M0 decode of every byte against 2^(e-127);
the scale exponent against an exact integer log2 of the block maximum on every
binade; exact round trip of blocks built on the grid (one element at +-4..6 so
the block's scale is the one used to build it); saturation between 6 and 8;
zero blocks; the blocked form of the product against the dequantized product.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .codec import e2m1_decode, e2m1_encode

F32 = np.float32
MX_GROUP = 32
E2M1_EMAX = 2


def e8m0_decode(e) -> np.ndarray:
    """E8M0 byte -> 2^(e - 127) as float64 (255 -> NaN)."""
    e = np.asarray(e, dtype=np.int64)
    out = np.ldexp(1.0, e - 127).astype(np.float64)
    return np.where(e == 255, np.nan, out)


def mx_scale_exponent(amax) -> np.ndarray:
    """X = floor(log2(amax)) - 2 for positive float32 amax, clamped to [-127, 127]; -127 for amax = 0."""
    a = np.asarray(amax, dtype=np.float32).astype(np.float64)
    _, e = np.frexp(a)                      # a = m 2^e, 0.5 <= m < 1 (exact for float32 inputs)
    X = np.where(a > 0, e - 1 - E2M1_EMAX, -127)
    return np.clip(X, -127, 127).astype(np.int64)


def mxfp4_quantize(T):
    """Quantize each row of T (float32, rows x K, K % 32 == 0) in blocks of 32 along K.

    Returns (codes uint8 rows x K, one E2M1 code per byte; scales uint8 rows x K/32, E8M0)."""
    T = np.asarray(T, dtype=np.float32)
    rows, K = T.shape
    if K % MX_GROUP:
        raise ValueError("K must be a multiple of 32")
    G = T.reshape(rows, K // MX_GROUP, MX_GROUP)
    a = np.abs(G).max(axis=2)
    X = mx_scale_exponent(a)
    q = np.ldexp(G.astype(np.float64), -X[:, :, None]).astype(np.float32)   # exact: a power of two
    codes = e2m1_encode(q)
    codes[a == 0] = 0
    return codes.reshape(rows, K), (X + 127).astype(np.uint8)


def mx_dequantize(codes, scales) -> np.ndarray:
    """code * 2^(e - 127) in float64 (exact)."""
    codes = np.asarray(codes)
    return e2m1_decode(codes) * e8m0_decode(scales).repeat(MX_GROUP, axis=1)


@dataclass
class MxPackedWeight:
    codes: np.ndarray      # N x K
    scales: np.ndarray     # N x K/32 E8M0


@dataclass
class MxQuantAct:
    codes: np.ndarray      # M x K
    scales: np.ndarray     # M x K/32
    LA: np.ndarray         # M x r float64: X L1f


def mx_pack_weight(R32) -> MxPackedWeight:
    """MXFP4 quantization of the residual R (K x N float32): blocks of 32 along K per column n."""
    codes, scales = mxfp4_quantize(np.ascontiguousarray(np.asarray(R32, dtype=np.float32).T))
    return MxPackedWeight(codes=codes, scales=scales)


def mx_quantize_act(X, inv_s, L1f: Optional[np.ndarray]) -> MxQuantAct:
    """X_hat = f32(X * inv_s), its MXFP4 codes, and X L1f in float64."""
    X = np.asarray(X, dtype=np.float64)
    xh = (X.astype(np.float32) * np.asarray(inv_s, dtype=np.float32)).astype(np.float32)
    codes, scales = mxfp4_quantize(xh)
    LA = X @ np.asarray(L1f, dtype=np.float64) if L1f is not None and L1f.shape[1] else np.zeros((X.shape[0], 0))
    return MxQuantAct(codes=codes, scales=scales, LA=LA)


def mx_linear(qa: MxQuantAct, pw: MxPackedWeight, L2b: Optional[np.ndarray], bias: Optional[np.ndarray]):
    """Y = sum_k dec(x) dec(w) + LA L2b + bias, float64."""
    Y = mx_dequantize(qa.codes, qa.scales) @ mx_dequantize(pw.codes, pw.scales).T
    if L2b is not None and L2b.shape[0]:
        Y = Y + qa.LA @ np.asarray(L2b, dtype=np.float64)
    if bias is not None:
        Y = Y + np.asarray(bias, dtype=np.float64)[None, :]
    return Y


def mx_reference(X, inv_s, L1f, L2b, R32, bias):
    """The whole MXFP4 layer: returns (Y float64, MxQuantAct, MxPackedWeight)."""
    pw = mx_pack_weight(R32)
    qa = mx_quantize_act(X, inv_s, L1f)
    return mx_linear(qa, pw, L2b, bias), qa, pw
