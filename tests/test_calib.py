"""The product's offline decomposition (calib.py, torch float64) against the oracle's
(oracle/decompose.py, numpy float64): two independent implementations of the same steps
("From SmoothQuant to SVDQuant", Smooth Quant (W8A8) and SVD decomposition; SVDQuant review §4.2)."""
import numpy as np
import pytest
import torch

from oracle import decompose as OD
from w4a4_rank_absorbed_b200.calib import calibrate
from w4a4_rank_absorbed_b200.synth import make_workload, small_case


def _bits_equal_fraction(a, b):
    a = np.asarray(a, dtype=np.float32).view(np.uint32)
    b = np.asarray(b, dtype=np.float32).view(np.uint32)
    return float(np.mean(a == b))


@pytest.mark.parametrize("case", [("small", 64, 256, 192, 16), ("small", 37, 512, 128, 32), ("tiny",),
                                  ("lora",)])
def test_calibration_matches_the_oracle(case):
    if case[0] == "small":
        _, M, K, N, r = case
        wl = small_case(M, K, N, r, seed=M + K + N)
    elif case[0] == "tiny":
        wl = make_workload("tiny")
    else:
        wl = small_case(48, 256, 160, 16, seed=9)
        rng = np.random.default_rng(3)
        wl.lora_A = rng.normal(0, 0.01, (wl.K, 16))
        wl.lora_B = rng.normal(0, 0.01, (16, wl.N))
    r = wl.r
    got = calibrate(wl.X, wl.W, r, wl.alpha, bias=wl.bias, lora_A=wl.lora_A, lora_B=wl.lora_B)
    dec = OD.decompose(wl.X, wl.W, r, wl.alpha, wl.lora_A, wl.lora_B)
    r_eff = dec.L1f.shape[1]
    assert got.r == r_eff
    # smoothing factors: float64 pow on both sides, then one rounding to float32
    assert _bits_equal_fraction(got.inv_s.numpy(), dec.inv_s) >= 0.99
    assert np.allclose(got.inv_s.numpy(), dec.inv_s, rtol=2 ** -23, atol=0)
    assert np.float32(got.gs_x) == dec.gs_x or abs(got.gs_x / float(dec.gs_x) - 1) <= 2 ** -23
    # the residual and the stored low-rank product are unique (sign choices of the SVD cancel)
    R_rel = np.linalg.norm(got.R.double().numpy() - dec.R32.astype(np.float64)) / np.linalg.norm(dec.R)
    assert R_rel <= 1e-6
    LL_got = got.L1fT.t().double().numpy() @ got.L2b.double().numpy()
    LL_or = dec.L1f @ dec.L2b
    assert np.linalg.norm(LL_got - LL_or) / np.linalg.norm(LL_or) <= 1e-3
    if wl.bias is not None:
        assert np.array_equal(got.bias.float().numpy(), torch.from_numpy(wl.bias).to(torch.bfloat16).float().numpy())


def test_randomized_range_finder_on_cpu_matches_truncated_svd():
    """The randomized split (the GPU calibration's algorithm; torch on the CPU here) against numpy's
    truncated SVD: same error to 1e-3 and the same leading singular values."""
    import torch
    from oracle import decompose as OD
    from w4a4_rank_absorbed_b200.calib import randomized_rank_r
    from w4a4_rank_absorbed_b200.synth import make_workload
    wl = make_workload("tiny")
    s = OD.smoothing_factors(wl.X, wl.W, wl.alpha)
    W_hat = s[:, None] * wl.W
    _, _, R, S = OD.low_rank_split(W_hat, 32)
    G1, G2 = randomized_rank_r(torch.from_numpy(W_hat), 32)
    err = float(torch.linalg.norm(torch.from_numpy(W_hat) - G1 @ G2))
    assert err <= np.linalg.norm(R) * (1 + 1e-3)
    sg = torch.linalg.svdvals(G1 @ G2).numpy()[:4]
    assert np.max(np.abs(sg - S[:4]) / S[:4]) <= 1e-8
