"""GPU-side calibration (svdq_calib_* kernels and calib.calibrate_gpu) against the oracle's decomposition."""
import numpy as np
import pytest
import torch

from helpers import GpuLayer, bf16_dev, oracle_layer, require_gpu
from oracle import decompose as OD
from oracle import linear as OL
from w4a4_rank_absorbed_b200.synth import make_workload, small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _C():
    from w4a4_rank_absorbed_b200 import svdq as C
    return C


def _err():
    st, site = _C().svdq_get_device_error()
    assert st == 0, site


@pytest.mark.parametrize("M,K", [(1000, 264), (37, 8), (4608, 3072), (1, 512)])
def test_activation_channel_maxima_exact_and_streamed(M, K):
    C = _C()
    wl = small_case(M, K, 16, 0, seed=M + K)
    X = bf16_dev(wl.X)
    amax = torch.full((K,), -1.0, dtype=torch.float32, device="cuda")
    C.svdq_calib_absmax_cols(X, M, K, amax)
    torch.cuda.synchronize()
    assert np.array_equal(amax.cpu().numpy().astype(np.float64), np.abs(wl.X).max(axis=0))
    # two batches merged by max give the maxima of the whole
    h = M // 2
    C.svdq_calib_absmax_cols(X[:h].contiguous(), h, K, amax)
    C.svdq_calib_absmax_cols(X[h:].contiguous(), M - h, K, amax, accumulate=True)
    torch.cuda.synchronize()
    assert np.array_equal(amax.cpu().numpy().astype(np.float64), np.abs(wl.X).max(axis=0))
    _err()


@pytest.mark.parametrize("M,K,N,alpha", [(512, 256, 384, 0.5), (300, 264, 100, 0.3), (4608, 3072, 9216, 0.5)])
def test_smoothing_and_scaled_weight_against_oracle(M, K, N, alpha):
    C = _C()
    wl = small_case(M, K, N, 0, seed=K + N)
    wl.W[5, :] = 0.0                                  # a zero weight row: s = 1 there
    X = bf16_dev(wl.X)
    W = torch.from_numpy(wl.W).cuda()
    ax = torch.empty(K, dtype=torch.float32, device="cuda")
    aw = torch.empty(K, dtype=torch.float64, device="cuda")
    s = torch.empty(K, dtype=torch.float64, device="cuda")
    inv_s = torch.empty(K, dtype=torch.float32, device="cuda")
    C.svdq_calib_absmax_cols(X, M, K, ax)
    C.svdq_calib_absmax_rows(W, K, N, aw)
    C.svdq_calib_smooth(ax, aw, K, alpha, s, inv_s)
    W_hat = torch.empty_like(W)
    C.svdq_calib_scale_rows(W, s, K, N, W_hat)
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    C.svdq_calib_act_amax(X, M, K, inv_s, amax)
    torch.cuda.synchronize()
    assert np.array_equal(aw.cpu().numpy(), np.abs(wl.W).max(axis=1))
    s_or = OD.smoothing_factors(wl.X, wl.W, alpha)
    s_g = s.cpu().numpy()
    assert s_g[5] == 1.0
    assert np.max(np.abs(s_g - s_or) / s_or) <= 1e-15          # two float64 pow calls and a division: a few ulp
    inv_or = (1.0 / s_or).astype(np.float32)
    inv_g = inv_s.cpu().numpy()
    ulps = np.abs(inv_g.view(np.int32).astype(np.int64) - inv_or.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1 and (ulps == 0).mean() > 0.999
    assert np.max(np.abs(W_hat.cpu().numpy() - s_or[:, None] * wl.W)) <= 4e-16 * np.abs(s_or[:, None] * wl.W).max()
    # the activation global scale: amax of f32(X inv_s), with the oracle's products on the GPU's factors'
    # exact twins (inv_s agrees on every element here, or the comparison is to one ulp of the maximum)
    xh_max = np.abs((wl.X.astype(np.float32) * inv_or).astype(np.float32)).max()
    if np.array_equal(inv_g, inv_or):
        assert float(amax.item()) == float(xh_max)
    else:
        assert abs(float(amax.item()) - float(xh_max)) <= float(xh_max) * 2.0 ** -23
    _err()


def test_randomized_split_is_near_the_truncated_svd():
    from w4a4_rank_absorbed_b200.calib import randomized_rank_r
    wl = make_workload("qkv", M=256)
    s = OD.smoothing_factors(wl.X, wl.W, wl.alpha)
    W_hat = s[:, None] * wl.W
    L1, L2, R, S = OD.low_rank_split(W_hat, 32)
    opt = np.linalg.norm(R)
    Wd = torch.from_numpy(W_hat).cuda()
    G1, G2 = randomized_rank_r(Wd, 32)
    err = float(torch.linalg.norm(Wd - G1 @ G2))
    assert err <= opt * (1 + 1e-3), (err, opt)
    # the leading directions (the outlier-driven singular values) are captured to high accuracy
    sg = torch.linalg.svdvals(G1 @ G2).cpu().numpy()[:8]
    assert np.max(np.abs(sg - S[:8]) / S[:8]) <= 1e-6


@pytest.mark.parametrize("name", ["tiny", "qkv"])
def test_gpu_calibrated_layer_keeps_the_method_effect(name):
    """A layer built from calibrate_gpu is as good as one built from the oracle's decomposition: its output
    error against the exact product X W (+ bias) is within 1% of the oracle-calibrated layer's."""
    from w4a4_rank_absorbed_b200.calib import calibrate_gpu
    wl = make_workload(name, M=512)
    exact = wl.X @ wl.W + wl.bias[None, :]
    dec = OD.decompose(wl.X, wl.W, wl.r, wl.alpha)
    g_or = GpuLayer(dec, wl.bias)
    Xd = bf16_dev(wl.X)
    Y_or = g_or.linear(*g_or.quantize(Xd), y_fp32=True).cpu().numpy().astype(np.float64)
    data = calibrate_gpu(wl.X, wl.W, wl.r, wl.alpha, bias=wl.bias)
    assert float(np.float32(dec.gs_x)) == pytest.approx(data.gs_x, rel=2.0 ** -22)
    from w4a4_rank_absorbed_b200.layer import SVDQLinear
    L = SVDQLinear(data)
    Y = L.forward(Xd, y_fp32=True).cpu().numpy().astype(np.float64)
    e_or = OL.rel_fro(Y_or, exact)
    e_gpu = OL.rel_fro(Y, exact)
    print(f"{name}: oracle-calibrated {e_or:.4e}, GPU-calibrated {e_gpu:.4e}")
    assert e_gpu <= 1.01 * e_or
    _err()
