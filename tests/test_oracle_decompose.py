"""Pins of the oracle's offline decomposition (CPU only)."""
import numpy as np
import pytest

from oracle import decompose as D
from oracle.layout import sf_bytes, sf_from_storage, sf_offsets, sf_to_storage
from w4a4_rank_absorbed_b200.synth import make_workload, small_case


@pytest.fixture(scope="module")
def tiny():
    wl = make_workload("tiny")
    return wl, D.decompose(wl.X, wl.W, wl.r, wl.alpha)


def test_smoothing_identity(tiny):
    wl, dec = tiny
    Xh = wl.X / dec.s[None, :]
    Wh = dec.s[:, None] * wl.W
    ref = wl.X @ wl.W
    assert np.linalg.norm(Xh @ Wh - ref) / np.linalg.norm(ref) < 1e-12


def test_smoothing_factor_formula_alpha_limits():
    # alpha = 1 moves all of max|X_j| into s_j; alpha = 0 gives 1 / max|W_j|
    wl = small_case(8, 32, 16, 4)
    s1 = D.smoothing_factors(wl.X, wl.W, 1.0)
    s0 = D.smoothing_factors(wl.X, wl.W, 0.0)
    np.testing.assert_allclose(s1, np.abs(wl.X).max(axis=0), rtol=0, atol=0)
    np.testing.assert_allclose(s0, 1.0 / np.abs(wl.W).max(axis=1), rtol=1e-15)
    X = wl.X.copy()
    X[:, 3] = 0
    assert D.smoothing_factors(X, wl.W, 0.5)[3] == 1.0


def test_residual_identity_and_eckart_young(tiny):
    wl, dec = tiny
    Wh = dec.s[:, None] * wl.W
    assert np.linalg.norm(dec.L1 @ dec.L2 + dec.R - Wh) / np.linalg.norm(Wh) < 1e-12
    S = dec.sigma
    r = wl.r
    np.testing.assert_allclose(np.linalg.norm(dec.R) ** 2, np.sum(S[r:] ** 2), rtol=1e-10)
    np.testing.assert_allclose(np.linalg.norm(dec.R, 2), S[r], rtol=1e-10)


def test_low_rank_against_eigendecomposition(tiny):
    # The rank-r product is unique when sigma_r > sigma_{r+1}; compute it from eigh(W^T W) instead.
    wl, dec = tiny
    Wh = dec.s[:, None] * wl.W
    lam, V = np.linalg.eigh(Wh.T @ Wh)
    Vr = V[:, np.argsort(lam)[::-1][: wl.r]]
    P = Wh @ Vr @ Vr.T
    assert dec.sigma[wl.r - 1] > dec.sigma[wl.r] * (1 + 1e-6)
    assert np.linalg.norm(dec.L1 @ dec.L2 - P) / np.linalg.norm(P) < 1e-9


def test_outliers_absorbed(tiny):
    # The pages expect the residual to carry less energy than the smoothed weight and the
    # magnified rows to move into the low-rank branch ("From SmoothQuant to SVDQuant", SVDQuant (W4A4)).
    wl, dec = tiny
    Wh = dec.s[:, None] * wl.W
    assert np.linalg.norm(dec.R) < np.linalg.norm(Wh)
    assert np.abs(dec.R).max() < np.abs(Wh).max()


def test_lora_concatenation():
    wl = make_workload("sweep_r16_lora", M=64)
    dec = D.decompose(wl.X, wl.W, wl.r, wl.alpha, wl.lora_A, wl.lora_B)
    assert dec.L1f.shape == (wl.K, 32) and dec.L2b.shape == (32, wl.N)
    # exact branch: X_hat L1 L2 = X L1s L2 + X A B  (before the bf16 rounding of the stored factors)
    Xh = wl.X / dec.s[None, :]
    lhs = Xh @ dec.L1 @ dec.L2
    rhs = Xh @ dec.L1[:, :16] @ dec.L2[:16] + wl.X @ wl.lora_A @ wl.lora_B
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(lhs) < 1e-12


def test_bf16_round():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -7, -3.0000001, 0.0])
    got = D.bf16_round(v)
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0 + 2 ** -6, 1.0 + 2 ** -7, -3.0, 0.0])


def test_sf_layout_is_a_bijection():
    for rows, K in [(128, 64), (200, 128), (256, 512), (1, 64)]:
        KS = K // 16
        off = sf_offsets(rows, KS).reshape(-1)
        assert len(np.unique(off)) == off.size
        assert off.max() < sf_bytes(rows, K)
        rng = np.random.default_rng(rows)
        s = rng.integers(0, 256, size=(rows, KS)).astype(np.uint8)
        buf = sf_to_storage(s)
        assert buf.size == sf_bytes(rows, K)
        np.testing.assert_array_equal(sf_from_storage(buf, rows, KS), s)
    # the first 512-byte tile: row r, column kk at (r%32)*16 + (r//32)*4 + kk
    o = sf_offsets(128, 4)
    assert o[0, 0] == 0 and o[1, 0] == 16 and o[32, 0] == 4 and o[33, 3] == 16 + 4 + 3 and o[127, 3] == 511
    assert sf_offsets(128, 8)[0, 4] == 512 and sf_offsets(256, 4)[128, 0] == 512


def test_activation_global_scale_hand_built():
    # f32(X * inv_s) is exact here (powers of two), and the largest magnitude sits at a known
    # negative entry of a column whose smoothing factor enlarges it: amax = 168 * 4 = 672 -> 672/2688 = 1/4.
    X = np.zeros((6, 32))
    X[:, :] = 1.5
    X[3, 5] = -168.0
    X[0, 7] = 500.0                      # larger raw value, but its channel is shrunk by 1/8
    inv_s = np.ones(32, dtype=np.float32)
    inv_s[5] = 4.0
    inv_s[7] = 0.125
    assert D.activation_global_scale(X, inv_s) == np.float32(0.25)
    # without the smoothing the raw maximum 500 would decide: 500/2688 is a different scale
    assert D.activation_global_scale(X, np.ones(32, dtype=np.float32)) != np.float32(0.25)
    # all-zero activations: scale 1
    assert D.activation_global_scale(np.zeros((4, 16)), np.ones(16, dtype=np.float32)) == np.float32(1.0)


def test_activation_global_scale_rounds_the_product_to_float32_first():
    # x = 2688 (a bf16 value), inv_s = 1 + 2^-20: the exact product 2688 + 10.5 * 2^-12 is a tie at
    # float32's spacing 2^-12 and rounds to 2688 + 10 * 2^-12, so gs_x must come from the product
    # rounded to float32 first, then divided by 2688.
    s = np.float32(1.0 + 2.0 ** -20)
    X = np.full((2, 16), 2688.0)
    from w4a4_rank_absorbed_b200.synth import round_to_bf16
    assert round_to_bf16(X[0, 0]) == X[0, 0]
    inv_s = np.full(16, s, dtype=np.float32)
    got = D.activation_global_scale(X, inv_s)
    # f32(2709 (1 + 2^-20)) = 2709 + 2709 * 2^-20 rounded to float32's spacing 2^-12 at 2709
    from fractions import Fraction
    exact = Fraction(2688) * (1 + Fraction(1, 2 ** 20))
    spacing = Fraction(1, 2 ** 12)
    k, rem = divmod(exact, spacing)
    if rem * 2 > spacing or (rem * 2 == spacing and k % 2 == 1):
        k += 1
    prod32 = k * spacing
    assert float(prod32) != float(exact)          # the rounding step matters in this case
    q = prod32 / 2688
    sp = Fraction(1, 2 ** 23)                      # q is in [1, 2)
    k2, rem2 = divmod(q, sp)
    if rem2 * 2 > sp or (rem2 * 2 == sp and k2 % 2 == 1):
        k2 += 1
    assert got == np.float32(float(k2 * sp))


def test_bf16_round_against_torch_conversion():
    """bf16 rounding of the oracle against torch's float32 -> bfloat16 conversion (round to nearest even),
    over random float32 bit patterns (normals, subnormals, values that overflow to infinity)."""
    import torch
    rng = np.random.default_rng(11)
    x = rng.integers(0, 2 ** 32, 1_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    sub = np.arange(0, 2 ** 23, 13, dtype=np.uint32).view(np.float32)
    edge = np.array([3.3895314e38, 3.4e38, -3.4e38, 0.0, -0.0, 2.0 ** -126, 2.0 ** -133, 1.5 * 2.0 ** -133],
                    dtype=np.float32)
    for v in (x[np.isfinite(x)], sub, -sub, edge):
        t = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
        o = D.bf16_round(v.astype(np.float64))
        assert np.array_equal(t, o)
        assert np.array_equal(np.signbit(t), np.signbit(o))
