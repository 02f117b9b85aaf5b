"""NVFP4 codec of the oracle (test infrastructure; see the package header).

What it states (SVDQuant review, §3 Quantization Preliminary): a tensor is
quantized as Q_X = round(X / s_X) with s_X = max|X| / q_max, and q_max = 6
for 4-bit floating point.  "From SmoothQuant to SVDQuant", section Personal
view, names the NVFP4 variant: groups of 16 values with a two-level scale.
The reading taken here (the pages leave the details open):

  * 4-bit codes are FP4 E2M1 (sign, 2 exponent bits, 1 mantissa bit); the
    eight magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6, so q_max = 6.
  * Each group of 16 consecutive values along the reduction axis K has one
    unsigned E4M3 (UE4M3) block scale; each tensor has one float32 global
    scale gs = amax / (6 * 448) (gs = 1 when amax = 0), so the block scales
    use the full UE4M3 range.
  * Per group, with a = max|x| over the group and c = 1 / (6 * gs):
        sb   = UE4M3(a * c)                (round to nearest even, saturate at 448)
        d    = dec(sb) * gs
        code = E2M1(x * (1 / d))           (round to nearest even, saturate at 6)
    and all codes are 0 when dec(sb) = 0.  round() is read as round to
    nearest with ties to the even code; X / s_X is taken as a product with
    the reciprocal.  Every one of these float32 operations is a single
    correctly rounded binary32 operation, the same sequence the kernels run.
  * The sign bit of a code is the sign bit of x * (1/d) (so a negative value
    that rounds to zero gives the code 0x8, "-0"), except in all-zero-scale
    groups, which emit 0x0.

Pins (tests/test_oracle_codec.py): E2M1 encode against an independent
binade-wise np.rint rounding on a dense sweep with every tie; UE4M3 encode
and decode against torch's float8_e4m3fn conversion (a library routine);
the 16-entry E2M1 table (tests/golden/e2m1_table.txt); exact round trip of
tensors built on the grid; saturation and zero-group special cases.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
Q_MAX = 6.0            # largest E2M1 magnitude (q_max of the 4-bit FP quantizer)
UE4M3_MAX = 448.0      # largest finite E4M3 magnitude
GS_DENOM = F32(Q_MAX * UE4M3_MAX)   # 2688


# ---------------------------------------------------------------- E2M1 -------
def e2m1_decode(codes) -> np.ndarray:
    """Value of each 4-bit E2M1 code (low nibble of ``codes``), float64."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode(q) -> np.ndarray:
    """Round float32 values to the nearest E2M1 code, ties to the even code, saturating at 6.

    Nearest-grid-point search: for each |q| find the grid magnitude at the
    least distance; when two are equally near, take the one whose code is
    even (its mantissa bit is 0).  Values beyond 6 saturate to 6.  The sign
    bit is copied from q.
    """
    q = np.asarray(q, dtype=np.float32)
    if np.isnan(q).any():
        raise ValueError("NaN has no E2M1 code")
    a = np.abs(q.astype(np.float64))
    flat = a.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    chunk = 1 << 20
    for s in range(0, flat.size, chunk):
        v = flat[s:s + chunk]
        dist = np.abs(v[:, None] - E2M1_MAGNITUDES[None, :])
        best = np.argmin(dist, axis=1)                     # first minimiser
        nxt = np.minimum(best + 1, 7)
        tie = (nxt != best) & (dist[np.arange(v.size), nxt] == dist[np.arange(v.size), best])
        best = np.where(tie & (best % 2 == 1), nxt, best)  # of two tied codes, the even one
        best = np.where(v >= Q_MAX, 7, best)
        out[s:s + chunk] = best
    sign = np.signbit(q).reshape(-1).astype(np.uint8) << 3
    return (out | sign).reshape(q.shape)


# --------------------------------------------------------------- UE4M3 -------
def _ue4m3_table() -> np.ndarray:
    vals = np.empty(256, dtype=np.float64)
    for b in range(256):
        e, m = (b >> 3) & 0xF, b & 7
        mag = m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        if (b & 0x7F) == 0x7F:
            mag = np.nan
        vals[b] = -mag if b & 0x80 else mag
    return vals


UE4M3_VALUES = _ue4m3_table()
_UE4M3_FINITE = UE4M3_VALUES[:0x7F]          # codes 0x00..0x7E, increasing, 0 .. 448


def ue4m3_decode(b) -> np.ndarray:
    """Value of each E4M3 byte (sign bit honoured; 0x7F/0xFF are NaN), float64."""
    return UE4M3_VALUES[np.asarray(b).astype(np.int64) & 0xFF]


def ue4m3_encode(v) -> np.ndarray:
    """Round non-negative float32 values to the nearest UE4M3 byte, ties to even, saturating at 448."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    if (v < 0).any() or np.isnan(v).any():
        raise ValueError("UE4M3 scales are non-negative and finite")
    hi = np.searchsorted(_UE4M3_FINITE, v, side="left")        # first grid value >= v
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    dl = v - _UE4M3_FINITE[lo]
    dh = _UE4M3_FINITE[hi] - v
    pick = np.where(dh < dl, hi, lo)
    tie = (dh == dl) & (hi != lo)
    pick = np.where(tie, np.where(hi % 2 == 0, hi, lo), pick)
    pick = np.where(_UE4M3_FINITE[hi] == v, hi, pick)           # exactly on the grid
    pick = np.where(v >= UE4M3_MAX, 0x7E, pick)
    return pick.astype(np.uint8)


# ------------------------------------------------------------ quantizer ------
def global_scale(amax) -> np.float32:
    """Per-tensor float32 scale gs = amax / 2688 (one rounding), or 1 when amax = 0."""
    amax = F32(amax)
    if not np.isfinite(amax):
        raise ValueError("non-finite amax")
    if amax == 0:
        return F32(1.0)
    return F32(amax / GS_DENOM)


def nvfp4_quantize(T, gs):
    """Quantize each row of T (float32, rows x K, K % 16 == 0) in groups of 16 along K.

    Returns (codes uint8 rows x K, one E2M1 code per byte; scales uint8 rows x K/16).
    Follows the per-group steps in this module's header, each a float32 operation.
    """
    T = np.asarray(T, dtype=np.float32)
    rows, K = T.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    gs = F32(gs)
    c = F32(F32(1.0) / F32(F32(Q_MAX) * gs))
    G = T.reshape(rows, K // 16, 16)
    a = np.abs(G).max(axis=2)                                   # exact
    sb = ue4m3_encode(F32(a * c))
    dsb = ue4m3_decode(sb).astype(np.float32)
    d = F32(dsb * gs)
    zero = sb == 0
    with np.errstate(divide="ignore"):
        rinv = np.where(zero, F32(0.0), F32(1.0) / np.where(zero, F32(1.0), d)).astype(np.float32)
    q = (G * rinv[:, :, None]).astype(np.float32)
    codes = e2m1_encode(q)
    codes[zero] = 0
    return codes.reshape(rows, K), sb


def dequantize(codes, scales, gs) -> np.ndarray:
    """code * dec(scale) * gs in float64 (exact: a few significant bits times a float32)."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    s = ue4m3_decode(scales).repeat(16, axis=1)
    return e2m1_decode(codes) * s * np.float64(F32(gs))


def pack_codes(codes) -> np.ndarray:
    """Two codes per byte along K: element 2j in the low nibble, 2j+1 in the high nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_codes(packed) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out
