"""The packed-layer API (SVDQLinear) on the GPU: device forward, host-buffer forward and the
streamed host-buffer path agree with each other bit for bit and with the oracle."""
import numpy as np
import pytest
import torch

from helpers import OL, GpuLayer, bf16_dev, check_y, oracle_layer, require_gpu
from w4a4_rank_absorbed_b200.synth import small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _layer(M, K, N, r, seed):
    from w4a4_rank_absorbed_b200.calib import calibrate
    from w4a4_rank_absorbed_b200.layer import SVDQLinear
    wl = small_case(M, K, N, r, seed=seed)
    data = calibrate(wl.X, wl.W, r, 0.5, bias=wl.bias)
    return wl, data, SVDQLinear(data, device=torch.device("cuda", 0))


def test_forward_matches_oracle_and_host_paths():
    M, K, N, r = 300, 512, 528, 32
    wl, data, L = _layer(M, K, N, r, seed=41)
    X = torch.from_numpy(wl.X.astype(np.float32)).to(torch.bfloat16)
    Y_dev = L.forward(X.cuda()).cpu()
    # oracle on the same layer constants (the layer's own decomposition, its packed weight)
    inv_s = data.inv_s.double().numpy()
    L1f = data.L1fT.t().float().double().numpy()
    L2b = data.L2b.float().double().numpy()
    Y_or, _, _ = OL.svdq_reference(X.float().double().numpy(), inv_s, data.gs_x, L1f, L2b,
                                   data.R.numpy(), data.bias.float().double().numpy())
    check_y(Y_dev.float().numpy().astype(np.float64), Y_or, bf16=True, what="layer forward")

    Xh = X.pin_memory()
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    Xd, Yd = torch.empty((M, K), dtype=torch.bfloat16, device="cuda"), torch.empty((M, N), dtype=torch.bfloat16,
                                                                                    device="cuda")
    L.forward_host(Xh, Yh, Xd, Yd)
    torch.cuda.synchronize()
    assert torch.equal(Yh, Y_dev)


def test_streamed_host_batches_match_forward():
    M, K, N, r = 256, 256, 272, 16
    wl, data, L = _layer(M, K, N, r, seed=43)
    g = torch.Generator().manual_seed(7)
    Xs = [(torch.randn((M, K), generator=g) * (1.0 + 0.5 * i)).to(torch.bfloat16) for i in range(5)]
    want = [L.forward(X.cuda()).cpu() for X in Xs]
    Xh = [X.pin_memory() for X in Xs]
    Yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in Xs]
    X_devs = [torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    Y_devs = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    L.forward_host_stream(Xh, Yh, X_devs, Y_devs)
    torch.cuda.synchronize()
    for i in range(len(Xs)):
        assert torch.equal(Yh[i], want[i]), f"batch {i}"
    from w4a4_rank_absorbed_b200 import svdq as C
    assert C.svdq_get_device_error()[0] == 0


def test_tensor_maps_are_cached_across_calls():
    """The second and later forward passes on the same buffers encode no tensor map; host time per call
    through the C ABI is printed (eager launches, no graph)."""
    import time
    from w4a4_rank_absorbed_b200 import svdq as C
    wl = small_case(256, 512, 512, 32, seed=5)
    dec = oracle_layer(wl, 32)
    g = GpuLayer(dec, wl.bias)
    X = bf16_dev(wl.X)
    Xq, SFx, LAs = g.quantize(X)
    Y = g.linear(Xq, SFx, LAs)
    torch.cuda.synchronize()
    h0, m0 = C.svdq_map_cache_stats()
    n = 200
    t0 = time.perf_counter()
    for _ in range(n):
        C.svdq_linear(Xq, SFx, float(g.gs_x), g.Wq, g.SFw, float(g.gs_w), LAs, g.L2p, g.r, g.bias, Y, 0, 256, 512, 512)
    t1 = time.perf_counter()
    torch.cuda.synchronize()
    h1, m1 = C.svdq_map_cache_stats()
    assert m1 == m0, "a repeated call encoded a tensor map again"
    assert h1 - h0 == 4 * n                      # Xq, Wq, LAs, L2p maps of every call
    print(f"svdq_linear host time per call through ctypes, cached maps: {(t1 - t0) / n * 1e6:.1f} us")
    g.check_errors()


def test_packed_layer_state_round_trip(tmp_path):
    """A packed layer saved with torch.save and rebuilt without packing gives identical outputs."""
    from w4a4_rank_absorbed_b200.calib import calibrate
    from w4a4_rank_absorbed_b200.layer import SVDQLinear
    wl = small_case(300, 512, 384, 32, seed=21)
    L = SVDQLinear(calibrate(wl.X, wl.W, 32, wl.alpha, bias=wl.bias))
    X = bf16_dev(wl.X)
    Y0 = L.forward(X)
    path = tmp_path / "layer.pt"
    torch.save(L.state_dict(), path)
    L2 = SVDQLinear.from_state_dict(torch.load(path), device="cuda")
    Y1 = L2.forward(X)
    torch.cuda.synchronize()
    assert torch.equal(Y0, Y1)
    with pytest.raises(ValueError):
        bad = L.state_dict()
        bad["Wq"] = bad["Wq"][:, :10]
        SVDQLinear.from_state_dict(bad, device="cuda")
