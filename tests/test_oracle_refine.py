"""Pins of the oracle's iterative residual refinement (CPU only)."""
import numpy as np

from oracle import decompose as D
from oracle import refine as RF
from w4a4_rank_absorbed_b200.synth import make_workload, small_case


def _w_hat(wl):
    s = D.smoothing_factors(wl.X, wl.W, wl.alpha)
    return s[:, None] * wl.W


def _projector_rank_r(T, r):
    """Best rank-r approximation of T from an eigendecomposition of T^T T (not np.linalg.svd)."""
    w, V = np.linalg.eigh(T.T @ T)
    Vr = V[:, np.argsort(w)[::-1][:r]]
    return T @ Vr @ Vr.T


def test_zero_steps_is_the_plain_split():
    wl = small_case(64, 128, 96, 8, seed=3)
    W_hat = _w_hat(wl)
    L1, L2, R, hist = RF.refine(W_hat, 8, 0)
    P1, P2, PR, _ = D.low_rank_split(W_hat, 8)
    assert len(hist) == 1
    np.testing.assert_allclose(L1 @ L2, P1 @ P2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(R, PR, rtol=0, atol=1e-12)


def test_each_step_is_the_rank_r_fit_of_what_the_residual_misses():
    wl = small_case(64, 128, 96, 8, seed=4)
    W_hat = _w_hat(wl)
    _, _, _, hist = RF.refine(W_hat, 8, 3)
    assert len(hist) == 4
    for k in range(1, 4):
        target = W_hat - RF.quantized_residual(hist[k - 1].R)
        np.testing.assert_allclose(hist[k].target, target, rtol=0, atol=0)
        want = _projector_rank_r(target, 8)
        L = hist[k].L1 @ hist[k].L2
        assert np.linalg.norm(L - want) <= 1e-9 * np.linalg.norm(want)
        np.testing.assert_allclose(hist[k].R, W_hat - L, rtol=0, atol=1e-12)
        # the kept error is || W_hat - L1 L2 - Q(R) || of that step
        assert abs(hist[k].error - RF.weight_error(W_hat, hist[k].L1, hist[k].L2, hist[k].R)) <= 1e-9


def test_kept_iterate_has_the_smallest_error():
    wl = small_case(64, 256, 128, 16, seed=5)
    W_hat = _w_hat(wl)
    L1, L2, R, hist = RF.refine(W_hat, 16, 4)
    errs = [h.error for h in hist]
    got = RF.weight_error(W_hat, L1, L2, R)
    assert abs(got - min(errs)) <= 1e-12 * max(errs)
    assert got <= errs[0]


def test_rank_zero_is_a_no_op():
    wl = small_case(32, 64, 48, 0, seed=6)
    W_hat = _w_hat(wl)
    L1, L2, R, hist = RF.refine(W_hat, 0, 2)
    assert L1.shape == (64, 0) and L2.shape == (0, 48)
    np.testing.assert_array_equal(R, W_hat)
    assert len({h.error for h in hist}) == 1


def test_refinement_lowers_the_weight_error_on_outlier_data():
    # The tiny FLUX-like recipe: a few magnified weight rows after smoothing.  The page's point is that
    # optimizing R repeatedly lowers the quantization error of the decomposition.
    wl = make_workload("tiny")
    W_hat = _w_hat(wl)
    _, _, _, hist = RF.refine(W_hat, 32, 3)
    assert min(h.error for h in hist[1:]) < hist[0].error
    dec0 = D.decompose(wl.X, wl.W, 32, wl.alpha)
    dec3 = D.decompose(wl.X, wl.W, 32, wl.alpha, refine_iters=3)
    e0 = RF.weight_error(W_hat, dec0.L1, dec0.L2, dec0.R)
    e3 = RF.weight_error(W_hat, dec3.L1, dec3.L2, dec3.R)
    assert e3 < e0
    # the smoothing identity and the split still hold for the refined decomposition
    np.testing.assert_allclose(dec3.L1 @ dec3.L2 + dec3.R, W_hat, rtol=0, atol=1e-9 * np.abs(W_hat).max())
