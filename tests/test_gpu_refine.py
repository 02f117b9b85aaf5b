"""Iterative refinement of the decomposition (SVDQuant review, section 4.2: R optimized repeatedly):
the library's dequantization of a packed weight, and the product's refinement loop, against the oracle."""
import numpy as np
import pytest
import torch

from helpers import OD, OL, check_y, f32_dev, require_gpu
from oracle import refine as RF
from w4a4_rank_absorbed_b200.synth import make_workload, small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("K,N", [(64, 16), (512, 400), (1024, 1040)])
def test_dequant_weight_matches_oracle(K, N):
    from w4a4_rank_absorbed_b200 import svdq as C
    rng = np.random.default_rng(K + N)
    R = (rng.standard_normal((K, N)) * 0.05).astype(np.float32)
    R[:, 3] *= 30.0
    R[5, :] = 0.0
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    SFw = torch.empty(C.svdq_sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    C.svdq_pack_weight(f32_dev(R), None, K, N, 0, Wq, SFw, gs, None)
    Rq = torch.empty((K, N), dtype=torch.float32, device="cuda")
    C.svdq_dequant_weight(Wq, SFw, gs, K, N, Rq)
    torch.cuda.synchronize()
    got = Rq.cpu().numpy().astype(np.float64)
    want = RF.quantized_residual(R)           # float64, exact value of the codes
    # two float32 roundings (the scale product, then the code times it)
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -22)
    assert C.svdq_get_device_error()[0] == 0


@pytest.mark.parametrize("name,M,iters", [("tiny", None, 3), ("qkv", 256, 2)])
def test_refined_decomposition_matches_oracle(name, M, iters):
    from w4a4_rank_absorbed_b200.calib import calibrate, refine_split
    wl = make_workload(name, M=M)
    if name == "qkv":           # a 512 x 768 corner of the QKV layer keeps the host SVDs quick
        wl.W = wl.W[:512, :768]
        wl.X = wl.X[:, :512]
        wl.bias = wl.bias[:768]
        wl.K, wl.N = 512, 768
    s = OD.smoothing_factors(wl.X, wl.W, wl.alpha)
    W_hat = s[:, None] * wl.W
    _, _, _, hist = RF.refine(W_hat, wl.r, iters)
    _, _, _, errs = refine_split(torch.from_numpy(W_hat), wl.r, iters, torch.device("cuda", 0))
    want = [h.error for h in hist]
    np.testing.assert_allclose(errs, want, rtol=1e-6)
    assert min(errs) < errs[0]
    # the refined layer runs through the library and matches the oracle on the same constants
    from w4a4_rank_absorbed_b200.layer import SVDQLinear
    data = calibrate(wl.X, wl.W, wl.r, wl.alpha, bias=wl.bias, refine_iters=iters, device="cuda")
    L = SVDQLinear(data, device=torch.device("cuda", 0))
    X = torch.from_numpy(wl.X.astype(np.float32)).to(torch.bfloat16)
    Y = L.forward(X.cuda(), y_fp32=True).cpu().numpy().astype(np.float64)
    Y_or, _, _ = OL.svdq_reference(X.double().numpy(), data.inv_s.double().numpy(), data.gs_x,
                                   data.L1fT.t().double().numpy(), data.L2b.double().numpy(), data.R.numpy(),
                                   data.bias.double().numpy())
    check_y(Y, Y_or, bf16=False, what=f"refined {name}")
