"""Pins of the oracle's GELU and MLP chain (oracle/mlp.py) against values fixed by mathematics."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import decompose as OD
from oracle import linear as OL
from oracle import mlp as OM
from w4a4_rank_absorbed_b200.synth import small_case


def _all_finite_bf16() -> np.ndarray:
    y = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    return y[np.isfinite(y)]


def _round_fraction_to_f32(x: Fraction) -> float:
    """Exact round-to-nearest-even of a rational to binary32 (normal and subnormal range)."""
    if x == 0:
        return 0.0
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()      # 2^(e-1) < x < 2^(e+1)
    while Fraction(2) ** e <= x:
        e += 1
    while Fraction(2) ** (e - 1) > x:
        e -= 1                                                       # 2^(e-1) <= x < 2^e
    q = max(e - 24, -149)                                            # spacing 2^q
    m = x / Fraction(2) ** q
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * float(Fraction(n) * Fraction(2) ** q)


def test_fma32_is_one_rounding_of_the_exact_value():
    rng = np.random.default_rng(3)
    a = rng.standard_normal(3000).astype(np.float32) * np.float32(3.0)
    b = rng.standard_normal(3000).astype(np.float32)
    c = rng.standard_normal(3000).astype(np.float32) * np.float32(0.5)
    # products whose low bits make a + b*c land on (or next to) binary32 midpoints
    k = np.arange(1, 400, dtype=np.float32)
    a2 = (np.float32(1.0) + k * np.float32(2.0 ** -12)).astype(np.float32)
    b2 = (np.float32(1.0) + np.float32(2.0 ** -12)) * np.ones_like(a2)
    c2 = np.where(np.arange(k.size) % 3 == 0, np.float32(2.0 ** -60),
                  np.where(np.arange(k.size) % 3 == 1, np.float32(-2.0 ** -60), np.float32(0.0))).astype(np.float32)
    tiny = np.array([1e-40, -1e-40, 3e-39], dtype=np.float32)          # subnormal results
    for A, B, Cc in ((a, b, c), (a2, b2, c2), (tiny, np.float32([0.5, 0.75, 1.5]), np.float32([1e-45, 0.0, -1e-45]))):
        got = OM.fma32(A, B, Cc)
        for i in range(A.size):
            exact = Fraction(float(A[i])) * Fraction(float(B[i])) + Fraction(float(Cc[i]))
            assert float(got[i]) == _round_fraction_to_f32(exact), (A[i], B[i], Cc[i])


def test_exp_against_float64_exponential():
    x = -np.linspace(0.0, 80.0, 400001).astype(np.float32)
    e = OM.exp_m80_0_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    assert np.max(np.abs(e - ref) / ref) <= 4.0 * 2.0 ** -24     # within 4 ulp of float32
    assert OM.exp_m80_0_f32(np.float32(0.0)) == 1.0
    with pytest.raises(ValueError):
        OM.exp_m80_0_f32(np.float32(1.0))
    with pytest.raises(ValueError):
        OM.exp_m80_0_f32(np.float32(-80.5))


def test_reciprocal_on_one_to_two():
    d = np.linspace(1.0, 2.0, 1000001).astype(np.float32)
    q = OM.recip_1_2(d).astype(np.float64)
    exact = 1.0 / d.astype(np.float64)
    assert np.max(np.abs(q - exact) / exact) <= 1.5 * 2.0 ** -24
    assert OM.recip_1_2(np.float32(1.0)) == 1.0 and OM.recip_1_2(np.float32(2.0)) == 0.5
    assert float(OM.R0A) == pytest.approx(24.0 / 17.0, rel=1e-7) and float(OM.R0B) == pytest.approx(8.0 / 17.0, rel=1e-7)


def test_taylor_coefficients_are_reciprocal_factorials():
    for k, c in enumerate(OM.TAYLOR):
        assert c == np.float32(1.0 / math.factorial(k))
    assert OM.C3 == np.float32(float(OM.C2) * 0.044715) or abs(float(OM.C3) / (float(OM.C2) * 0.044715) - 1) < 1e-7
    assert float(OM.LN2_HI) + float(OM.LN2_LO) == pytest.approx(math.log(2.0), rel=1e-15, abs=1e-12)
    assert float(OM.LN2_HI) * 65536.0 == int(float(OM.LN2_HI) * 65536.0)    # 16 significant bits


def test_gelu_f32_against_logistic_form_on_every_bf16_input():
    y = _all_finite_bf16()
    g = OM.gelu_f32(y).astype(np.float64)
    c = OM.gelu_logistic_f64(y.astype(np.float64))
    with np.errstate(over="ignore"):
        t = np.abs(2.0 * np.sqrt(2.0 / np.pi) * (y.astype(np.float64) + 0.044715 * y.astype(np.float64) ** 3))
    # exp(-|t|) turns the relative rounding of t into |t| times as much: the bound grows with |t|;
    # below exp(-80) the exponential is cut to zero (|GELU| < 2e-33 there).
    bound = 6.0 * 2.0 ** -24 * (2.0 + np.minimum(t, 1e30)) * np.abs(c) + 2e-33
    assert np.all(np.abs(g - c) <= bound)


def test_logistic_form_equals_the_tanh_closed_form_and_torch():
    y = np.linspace(-3.0, 3.0, 6001)
    c = OM.gelu_logistic_f64(y)
    assert np.max(np.abs(c - OM.gelu_closed_form(y))) <= 1e-14
    t = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    assert np.max(np.abs(c - t)) <= 1e-14
    # a wrong constant would move these by far more than the rounding
    assert abs(OM.gelu_logistic_f64(1.0) - 0.8411919906082768) < 1e-15
    assert abs(OM.gelu_logistic_f64(-1.0) - (-0.15880800939172324)) < 1e-15
    assert float(OM.gelu_f32(np.float32(1.0))) == pytest.approx(0.8411919906082768, rel=3e-7)


def test_gelu_special_values_and_odd_part():
    z = OM.gelu_f32(np.array([0.0, -0.0, 1e30, -1e30, 3.0e38, -3.0e38], dtype=np.float32))
    assert z[0] == 0.0 and not np.signbit(z[0])
    assert z[1] == 0.0 and np.signbit(z[1])
    assert z[2] == np.float32(1e30) and z[3] == 0.0
    assert z[4] == np.float32(3.0e38) and z[5] == 0.0
    y = np.linspace(0.0, 9.0, 9001).astype(np.float32)
    odd = OM.gelu_f32(y).astype(np.float64) - OM.gelu_f32(-y).astype(np.float64)
    assert np.max(np.abs(odd - y.astype(np.float64))) <= 4 * 2.0 ** -24 * (1.0 + y.max())


def test_gelu_bf16_is_the_rounded_gelu():
    y = _all_finite_bf16().astype(np.float64)
    gb = OM.gelu_bf16(y)
    cb = OD.bf16_round(OM.gelu_logistic_f64(y))
    assert np.array_equal(gb, OD.bf16_round(gb))                      # bf16 values
    same = gb == cb
    # away from the exp cut-off (y > -9.5) they differ only where the float32 value sits at a tie
    assert same[y > -9.5].mean() > 0.9995
    spacing = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(cb), 1e-38))) - 7)
    assert np.all(np.abs(gb - cb)[y > -9.5] <= spacing[y > -9.5])


def test_chain_against_its_parts_element_by_element():
    wl1 = small_case(5, 64, 32, 16, seed=3)
    dec1 = OD.decompose(wl1.X, wl1.W, 16, wl1.alpha)
    Y1, _, _ = OL.svdq_reference(wl1.X, dec1.inv_s, dec1.gs_x, dec1.L1f, dec1.L2b, dec1.R32, wl1.bias)
    W2 = np.random.default_rng(7).normal(0, 0.02, size=(32, 16))
    x2_guess = OM.gelu_bf16(OD.bf16_round(Y1))
    dec2 = OD.decompose(x2_guess, W2, 16, 0.5)
    c = OM.fc2_input(Y1, dec2.inv_s, dec2.gs_x, dec2.L1f)
    for i in range(Y1.shape[0]):
        for j in range(Y1.shape[1]):
            y1 = OD.bf16_round(np.float64(Y1[i, j]))
            assert c.y1[i, j] == y1
            ref = OM.gelu_logistic_f64(y1)
            assert abs(c.x2[i, j] - ref) <= 2.0 ** -8 * abs(ref) + 1e-30     # within a bf16 rounding
    qa = OL.quantize_act(c.x2, dec2.inv_s, dec2.gs_x, dec2.L1f)
    assert np.array_equal(qa.codes, c.qa2.codes) and np.array_equal(qa.scales, c.qa2.scales)
    assert np.allclose(c.qa2.LA, c.x2 @ dec2.L1f, rtol=0, atol=1e-12)
