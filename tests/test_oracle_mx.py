"""Pins of the oracle's MXFP4 codec and layer (CPU only)."""
from fractions import Fraction

import numpy as np

from oracle import codec as OC
from oracle import linear as OL
from oracle import mx as MX

F32 = np.float32


def _floor_log2(q: Fraction) -> int:
    n = q.numerator.bit_length() - q.denominator.bit_length()
    while Fraction(2) ** n > q:
        n -= 1
    while Fraction(2) ** (n + 1) <= q:
        n += 1
    return n


def test_e8m0_decode_every_byte():
    got = MX.e8m0_decode(np.arange(256))
    for e in range(255):
        assert Fraction(float(got[e])) == Fraction(2) ** (e - 127)
    assert np.isnan(got[255])


def test_scale_exponent_against_exact_log2():
    vals = []
    for n in range(-140, 127):
        p = 2.0 ** n
        vals += [p, np.nextafter(F32(p), F32(0)), F32(p) * F32(1.5)]
    rng = np.random.default_rng(2)
    vals += list(np.exp(rng.uniform(-80, 80, 3000)))
    a = np.array([v for v in vals if 0 < v < 3.0e38], dtype=F32)
    X = MX.mx_scale_exponent(a)
    for v, x in zip(a, X):
        want = max(-127, min(127, _floor_log2(Fraction(float(v))) - 2))
        assert x == want, (v, x, want)
    assert MX.mx_scale_exponent(F32(0.0)) == -127


def _grid_blocks(rng, rows, K):
    G = K // 32
    X = rng.integers(-100, 100, size=(rows, G))
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    cg = codes.reshape(rows, G, 32)
    hit = rng.integers(0, 32, size=(rows, G))
    top = rng.choice([6, 7], size=(rows, G)) | (rng.integers(0, 2, size=(rows, G)) << 3)
    cg[np.arange(rows)[:, None], np.arange(G)[None, :], hit] = top          # |x| of 4 or 6 sets the scale
    vals = OC.e2m1_decode(codes).reshape(rows, G, 32) * np.ldexp(1.0, X)[:, :, None]
    return vals.reshape(rows, K).astype(F32), codes, (X + 127).astype(np.uint8)


def test_round_trip_of_values_on_the_grid():
    rng = np.random.default_rng(3)
    T, codes, scales = _grid_blocks(rng, 40, 256)
    got_c, got_s = MX.mxfp4_quantize(T)
    np.testing.assert_array_equal(got_s, scales)
    # -0 and +0 both decode to 0: compare values, and codes wherever the value is non-zero
    nz = OC.e2m1_decode(codes) != 0
    np.testing.assert_array_equal(got_c[nz], codes[nz])
    np.testing.assert_array_equal(MX.mx_dequantize(got_c, got_s), T.astype(np.float64))


def test_saturation_ties_and_zero_blocks():
    T = np.zeros((3, 32), dtype=F32)
    T[0, :4] = [7.5, 7.0, 6.5, -5.0]            # amax 7.5: scale 2^0, values above 6 saturate, 5 ties to 4
    T[1, :3] = [0.75, 0.5, -0.25]               # amax 0.75: scale 2^-3 -> 6, 4, -2
    c, s = MX.mxfp4_quantize(T)
    assert s[0, 0] == 127 and list(OC.e2m1_decode(c[0, :4])) == [6.0, 6.0, 6.0, -4.0]
    assert s[1, 0] == 127 - 3 and list(OC.e2m1_decode(c[1, :3])) == [6.0, 4.0, -2.0]
    assert s[2, 0] == 0 and not c[2].any()     # all-zero block


def test_blocked_product_equals_dequantized_product():
    rng = np.random.default_rng(4)
    A = rng.standard_normal((7, 96)).astype(F32) * 3
    B = rng.standard_normal((5, 96)).astype(F32) * 0.01
    ca, sa = MX.mxfp4_quantize(A)
    cb, sb = MX.mxfp4_quantize(B)
    want = MX.mx_dequantize(ca, sa) @ MX.mx_dequantize(cb, sb).T
    got = np.zeros_like(want)
    for i in range(7):
        for j in range(5):
            for g in range(3):
                sl = slice(32 * g, 32 * g + 32)
                dot = float(np.dot(OC.e2m1_decode(ca[i, sl]), OC.e2m1_decode(cb[j, sl])))
                got[i, j] += dot * 2.0 ** (int(sa[i, g]) - 127 + int(sb[j, g]) - 127)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)


def test_mx_is_coarser_than_nvfp4_on_gaussian_data():
    # Loose sanity (reported shape of the formats, not a pin of a value): with one power-of-two scale per
    # 32 values MXFP4 loses more than NVFP4's fine scale per 16 on the same Gaussian matrix.
    rng = np.random.default_rng(5)
    T = rng.standard_normal((256, 512)).astype(F32)
    c, s = MX.mxfp4_quantize(T)
    e_mx = np.linalg.norm(MX.mx_dequantize(c, s) - T) / np.linalg.norm(T)
    e_nv = np.linalg.norm(OL.fake_quant(T) - T) / np.linalg.norm(T)
    assert e_nv < e_mx < 0.25
