"""The MLP pair fc1 -> GELU -> fc2 in the oracle (test infrastructure; see the package header).

The pages apply the SVDQuant layer to every linear layer of a diffusion
transformer; its MLP is fc1, a GELU, then fc2 ("SVDQuant: Absorbing Outliers
by Low-Rank Components for 4-Bit Diffusion Models", abstract: FLUX.1;
"From SmoothQuant to SVDQuant", section SVDQuant (W4A4)).  §4.3 of the
SVDQuant review fuses each layer's low-rank down-projection into its
activation quantization so that the 16-bit activations are read once; the
fused MLP chain carries the same idea one step further: fc1's output tile
goes through the GELU and is quantized as fc2's activations without being
written out.  The pages define neither the activation nor the chain; the
readings taken here:

  * The activation is the tanh form of GELU,
        GELU(y) = 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))),
    computed in the equivalent logistic form y * sigma(2u),
    u = sqrt(2/pi) (y + 0.044715 y^3), which has no cancellation for y < 0.
  * Its input is fc1's output as a bf16 tensor (the value an unfused fc1
    writes), its output is rounded once to bf16 (the value an unfused GELU
    writes, and what fc2's quantizer reads).
  * The arithmetic is a fixed sequence of IEEE binary32 operations, each
    correctly rounded (a fused multiply-add fma(a, b, c) = a*b + c rounded
    once), so that a GPU kernel that performs the same operations
    reproduces it bit for bit (the quantizer's decisions then agree).  exp
    is evaluated for arguments in [-80, 0] by the Cody-Waite range
    reduction (W. J. Cody and W. Waite, "Software Manual for the Elementary
    Functions", 1980: x = n ln2 + f, ln2 split into a short high part and a
    low part) and the Taylor polynomial of e^f to degree 6 (|f| <= ln2/2:
    truncation below 1.2e-7 relative); 1/(1 + e) by Newton's iteration.

  gelu_f32(y):
      y2 = y*y;  h = fma(C3, y2, C2);  t = y*h                (t = 2u)
      x = -|t|
      a = fma(x, LOG2E, 1.5 2^23);  nf = a - 1.5 2^23        (nf = rint(x log2 e))
      f = fma(-nf, LN2_HI, x);  f = fma(-nf, LN2_LO, f)
      p = 1/6!;  p = fma(p, f, 1/k!) for k = 5 .. 0
      e = p * 2^nf  if x >= -80, else 0                      (e = exp(x))
      d = 1 + e                                              (in [1, 2])
      q = fma(-R0B, d, R0A), then three times: r = fma(-d, q, 1); q = fma(q, r, q)
          (Newton's iteration for 1/d from a linear seed of relative error
          at most 1/17: R0A = f32(24/17), R0B = f32(8/17))
      sigma = q if t >= 0 else e*q
      g = y*sigma
  with C2 = f32(2 sqrt(2/pi)), C3 = f32(C2 * 0.044715).

  fc1 -> fc2 chain:  Y1 (float64, the layer of oracle.linear) -> y1 = bf16(Y1)
      -> x2 = bf16(gelu_f32(y1)) -> fc2's activation quantization and
      low-rank down-projection (oracle.linear.quantize_act) -> fc2's layer.

Pins (tests/test_oracle_mlp.py): fma32 against the exact rational value
rounded once (random triples, binary32 midpoints approached from both sides,
subnormal results); exp against the float64 exponential over [-80, 0]
(within 4 float32 ulp); the reciprocal against 1/d over [1, 2] (within 1.5
ulp); gelu_f32 against the float64 logistic form over every finite bf16 input
(the bound grows with |t|, since exp(-|t|) magnifies the rounding of t); the
logistic form against the tanh closed form and torch's float64 GELU (tanh
approximation); GELU(+-1) against their decimal values; GELU(0) = 0 and
GELU(-0) = -0; the odd-part identity GELU(y) - GELU(-y) = y; the chain
against its parts on a tiny case computed element by element.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import decompose as OD
from . import linear as OL

F32 = np.float32

LOG2E = F32(1.4426950408889634)
LN2_HI = F32(0.693145751953125)            # 16 significant bits: n * LN2_HI is exact for |n| < 256
LN2_LO = F32(0.6931471805599453 - 0.693145751953125)
MAGIC = F32(12582912.0)                    # 1.5 * 2^23: adding it rounds to an integer
EXP_MIN_ARG = F32(-80.0)
R0A = F32(24.0 / 17.0)
R0B = F32(8.0 / 17.0)
C2 = F32(2.0 * np.sqrt(2.0 / np.pi))
C3 = F32(2.0 * np.sqrt(2.0 / np.pi) * 0.044715)
TAYLOR_DEGREE = 6


def _taylor_coeffs():
    c = []
    f = 1.0
    for k in range(8):
        if k:
            f *= k
        c.append(F32(1.0 / f))
    return c


TAYLOR = _taylor_coeffs()


def fma32(a, b, c) -> np.ndarray:
    """a*b + c rounded once to binary32 (round to nearest even), for binary32 a, b, c.

    a*b is exact in float64 (48 significant bits); s = a*b + c is rounded to float64 with its
    exact error err (TwoSum).  Rounding s to binary32 gives the right answer except when s sits
    exactly on a binary32 midpoint (binary32 midpoints are float64 numbers, so rounding to float64
    can land on one but not cross it); there the exact value lies on err's side."""
    A = np.asarray(a, dtype=F32).astype(np.float64)
    B = np.asarray(b, dtype=F32).astype(np.float64)
    C = np.asarray(c, dtype=F32).astype(np.float64)
    p = A * B
    with np.errstate(over="ignore", invalid="ignore"):
        s = p + C
        bb = s - p
        err = (p - (s - bb)) + (C - bb)
        r = s.astype(F32)
        other = np.where(r.astype(np.float64) < s, np.nextafter(r, F32(np.inf)), np.nextafter(r, F32(-np.inf)))
        mid = (s == (r.astype(np.float64) + other.astype(np.float64)) / 2.0) & np.isfinite(s)
        fix = mid & (err != 0)
        toward_up = err > 0
        pick = np.where(toward_up, np.maximum(r, other), np.minimum(r, other))
    return np.where(fix, pick, r).astype(F32)


def exp_m80_0_f32(x) -> np.ndarray:
    """e^x for float32 x in [-80, 0] by the binary32 sequence in the module header."""
    x = np.asarray(x, dtype=F32)
    if np.any(x > 0) or np.any(x < EXP_MIN_ARG):
        raise ValueError("exp_m80_0_f32 takes -80 <= x <= 0")
    a = fma32(x, LOG2E, MAGIC)
    nf = a - MAGIC
    f = fma32(-nf, LN2_HI, x)
    f = fma32(-nf, LN2_LO, f)
    p = np.full_like(f, TAYLOR[TAYLOR_DEGREE])
    for k in range(TAYLOR_DEGREE - 1, -1, -1):
        p = fma32(p, f, TAYLOR[k])
    return (p * np.ldexp(F32(1.0), nf.astype(np.int32)).astype(F32)).astype(F32)


def recip_1_2(d) -> np.ndarray:
    """1/d for float32 d in [1, 2]: Newton's iteration from a linear seed, the sequence in the module header."""
    d = np.asarray(d, dtype=F32)
    q = fma32(-R0B, d, R0A)
    for _ in range(3):
        r = fma32(-d, q, F32(1.0))
        q = fma32(q, r, q)
    return q


def gelu_f32(y) -> np.ndarray:
    """GELU (tanh form) of float32 y by the binary32 sequence in the module header."""
    y = np.asarray(y, dtype=F32)
    with np.errstate(over="ignore", invalid="ignore"):   # |y| > 2^64: y^2 overflows, t = +-inf
        y2 = y * y
        h = fma32(C3, y2, C2)
        t = y * h
    x = (-np.abs(t)).astype(F32)
    e = np.where(x < EXP_MIN_ARG, F32(0.0), exp_m80_0_f32(np.maximum(x, EXP_MIN_ARG))).astype(F32)
    d = F32(1.0) + e
    q = recip_1_2(d)
    sigma = np.where(t >= 0, q, e * q).astype(F32)
    return (y * sigma).astype(F32)


def gelu_bf16(y_bf16) -> np.ndarray:
    """bf16(gelu_f32(y)) for bf16-exact inputs (given as float64), returned as float64."""
    y = np.asarray(y_bf16, dtype=np.float64)
    g = gelu_f32(y.astype(F32)).astype(np.float64)
    return OD.bf16_round(g)


def gelu_logistic_f64(y) -> np.ndarray:
    """The logistic form y * sigma(2u) in float64 (no cancellation for y < 0)."""
    y = np.asarray(y, dtype=np.float64)
    with np.errstate(over="ignore"):
        t = 2.0 * np.sqrt(2.0 / np.pi) * (y + 0.044715 * y ** 3)
    e = np.exp(-np.abs(t))
    return y * np.where(t >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def gelu_closed_form(y) -> np.ndarray:
    """The float64 closed form 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))."""
    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (y + 0.044715 * y ** 3)))


@dataclass
class ChainFc2Input:
    y1: np.ndarray          # M x N1: bf16(Y1), float64
    x2: np.ndarray          # M x N1: bf16(GELU(y1)), float64 (fc2's activations)
    qa2: OL.QuantAct        # fc2's codes, scales and X2 L1f2


def fc2_input(Y1, inv_s2, gs_x2, L1f2: Optional[np.ndarray]) -> ChainFc2Input:
    """What the fused fc1 epilogue produces from fc1's float64 output Y1: fc2's quantized activations."""
    y1 = OD.bf16_round(np.asarray(Y1, dtype=np.float64))
    x2 = gelu_bf16(y1)
    return ChainFc2Input(y1=y1, x2=x2, qa2=OL.quantize_act(x2, inv_s2, gs_x2, L1f2))


def mlp_reference(X, dec1, bias1, dec2, bias2):
    """fc1 -> GELU -> fc2 with both layers as in oracle.linear.  Returns (Y2 float64, ChainFc2Input, Y1)."""
    Y1, _, _ = OL.svdq_reference(X, dec1.inv_s, dec1.gs_x, dec1.L1f, dec1.L2b, dec1.R32, bias1)
    c = fc2_input(Y1, dec2.inv_s, dec2.gs_x, dec2.L1f)
    pw2 = OL.pack_weight(dec2.R32)
    Y2 = OL.linear(c.qa2, dec2.gs_x, pw2, dec2.L2b, bias2)
    return Y2, c, Y1
