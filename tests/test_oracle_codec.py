"""Pins of the oracle's NVFP4 codec against things other than itself (CPU only)."""
import os

import numpy as np
import pytest
import torch

from oracle import codec
from oracle.codec import (e2m1_decode, e2m1_encode, global_scale, nvfp4_quantize, ue4m3_decode,
                          ue4m3_encode)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_table.txt")
F32 = np.float32


def _golden():
    codes, ties = {}, []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, a, b = line.split()
        if kind == "code":
            codes[int(a, 16)] = float(b)
        else:
            ties.append((float(a), int(b, 16)))
    return codes, ties


def test_e2m1_table_matches_golden():
    codes, ties = _golden()
    assert sorted(codes) == list(range(16))
    for c, v in codes.items():
        got = e2m1_decode(np.array([c]))[0]
        assert got == v and np.signbit(got) == np.signbit(v), (c, got, v)
    for x, c in ties:
        assert e2m1_encode(np.array([x], dtype=F32))[0] == c, (x, c)


def _e2m1_by_binade(v):
    """Independent rounding: integer rint (half to even) at each binade's quantum."""
    a = np.abs(v.astype(np.float64))
    out = np.where(a < 2, np.rint(2 * a) / 2,
                   np.where(a < 4, np.rint(a), np.minimum(2 * np.rint(a / 2), 6.0)))
    idx = np.searchsorted(codec.E2M1_MAGNITUDES, out)
    assert np.all(codec.E2M1_MAGNITUDES[idx] == out)
    return idx.astype(np.uint8) | (np.signbit(v).astype(np.uint8) << 3)


def test_e2m1_encode_against_binade_rounding():
    grid = np.arange(-8 * 256, 8 * 256 + 1, dtype=np.float64) / 256.0      # every tie, every grid point
    rng = np.random.default_rng(0)
    rnd = rng.standard_normal(200_000) * 3
    big = np.array([7.0, 8.0, 1e6, 3e38, -7.5, -1e30])
    v = np.concatenate([grid, rnd, big]).astype(F32)
    np.testing.assert_array_equal(e2m1_encode(v), _e2m1_by_binade(v))


def test_ue4m3_decode_against_torch():
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = ue4m3_decode(np.arange(256))
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert ue4m3_decode(np.array([0x7E]))[0] == 448.0


def test_ue4m3_encode_against_torch():
    vals = codec.UE4M3_VALUES[:0x7F]
    mids = (vals[:-1] + vals[1:]) / 2                      # every tie between neighbours
    rng = np.random.default_rng(1)
    rnd = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(464.0), 300_000))
    v = np.concatenate([vals, mids, rnd, [0.0, 2.0 ** -10, 2.0 ** -10 * 1.0001, 464.0]]).astype(F32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ue4m3_encode(v), ref)


def test_ue4m3_saturates():
    v = np.array([448.0, 460.0, 464.0, 464.01, 480.0, 1e6, 3e38], dtype=F32)
    assert (ue4m3_encode(v) == 0x7E).all()


def _nearest_f32(q):
    """The float32 nearest to the positive rational q (ties to even), found by exact rational search."""
    from fractions import Fraction
    q = Fraction(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    ulp = Fraction(2) ** (max(e, -126) - 23)           # normal (or subnormal) spacing at q
    k, rem = divmod(q, ulp)
    if rem * 2 > ulp or (rem * 2 == ulp and k % 2 == 1):
        k += 1
    return F32(float(k * ulp))


def test_global_scale_closed_forms():
    # amax = 2688 * 2^k gives exactly 2^k; 2688 = 21 * 2^7, so amax = 21 gives 2^-7
    for k in range(-30, 31):
        assert global_scale(F32(2688.0 * 2.0 ** k)) == F32(2.0 ** k)
    assert global_scale(F32(21.0)) == F32(2.0 ** -7)
    assert global_scale(F32(8064.0)) == F32(3.0)
    assert global_scale(0.0) == F32(1.0)
    with pytest.raises(ValueError):
        global_scale(np.inf)


def test_global_scale_is_the_correctly_rounded_quotient():
    from fractions import Fraction
    rng = np.random.default_rng(5)
    amaxes = np.concatenate([[F32(3.0), F32(7.0), F32(1e-30), F32(6.0e4)],
                             np.exp(rng.uniform(-20, 20, 2000)).astype(F32)])
    for a in amaxes:
        want = _nearest_f32(Fraction(float(a)) / 2688)
        assert global_scale(a) == want, (a, global_scale(a), want)


def _grid_tensor(rng, rows, K, gs):
    """Rows built on the grid: value = code * dec(sb) * gs, one element per group at +-6."""
    G = K // 16
    sb = rng.integers(1, 0x7F, size=(rows, G)).astype(np.uint8)
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    hit = rng.integers(0, 16, size=(rows, G))
    sgn = rng.integers(0, 2, size=(rows, G)).astype(np.uint8) << 3
    cg = codes.reshape(rows, G, 16)
    cg[np.arange(rows)[:, None], np.arange(G)[None, :], hit] = 0x7 | sgn
    T = e2m1_decode(codes) * ue4m3_decode(sb).repeat(16, axis=1) * float(gs)
    T32 = T.astype(F32)
    assert np.array_equal(T32.astype(np.float64), T)          # exactly representable
    return T32, codes, sb


@pytest.mark.parametrize("gs", [2.0 ** -3, 2.0 ** -9, 1.0, 2.0 ** 4])
def test_quantizer_round_trip_on_grid(gs):
    rng = np.random.default_rng(int(np.log2(gs)) + 20)
    T, codes, sb = _grid_tensor(rng, 64, 256, gs)
    got_c, got_s = nvfp4_quantize(T, F32(gs))
    np.testing.assert_array_equal(got_s, sb)
    np.testing.assert_array_equal(got_c, codes)


def test_quantizer_zero_group_and_negative_zero():
    T = np.zeros((2, 32), dtype=F32)
    T[1, :16] = -0.0
    T[1, 16] = 3.0
    T[1, 17] = -1e-9                  # rounds to zero under a scale of 3/6
    c, s = nvfp4_quantize(T, F32(1.0))
    assert (c[0] == 0).all() and (s[0] == 0).all()
    assert (c[1, :16] == 0).all() and s[1, 0] == 0          # all-zero group emits 0x0, even for -0
    assert c[1, 16] == 0x7 and c[1, 17] == 0x8              # -tiny -> "-0"
    assert (c[1, 18:] == 0).all()


def test_quantizer_scale_rounded_down_saturates():
    # a/6 = 1.0625 is the tie between UE4M3 1.0 and 1.125; ties go to the even code (1.0),
    # so a / d = 6.375 saturates to the code for 6.
    T = np.zeros((1, 16), dtype=F32)
    T[0, 0] = 6.375
    T[0, 1] = -6.375
    T[0, 2] = 5.0                      # 5 is the tie between 4 and 6 -> 4 (even code 0x6)
    c, s = nvfp4_quantize(T, F32(1.0))
    assert ue4m3_decode(s)[0, 0] == 1.0
    assert c[0, 0] == 0x7 and c[0, 1] == 0xF and c[0, 2] == 0x6


def test_quantizer_saturating_scale():
    # a * c beyond 448 (a calibration scale too small for this group): scale saturates at 448
    T = np.full((1, 16), 5000.0, dtype=F32)
    c, s = nvfp4_quantize(T, F32(1.0))
    assert s[0, 0] == 0x7E and (c == 0x7).all()


def test_pack_unpack():
    rng = np.random.default_rng(3)
    c = rng.integers(0, 16, size=(5, 64)).astype(np.uint8)
    p = codec.pack_codes(c)
    assert p.shape == (5, 32)
    assert p[0, 0] == (c[0, 0] | (c[0, 1] << 4))
    np.testing.assert_array_equal(codec.unpack_codes(p), c)
