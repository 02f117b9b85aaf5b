"""Parity of the CUDA path against the oracle at small sizes (several tiles, ragged tails, edge cases)."""
import numpy as np
import pytest
import torch

from helpers import (GpuLayer, OC, OD, OL, bf16_dev, bf16_host, check_las, check_y, las_join,
                     mismatch_report, oracle_layer, oracle_storage, require_gpu, u8_host)
from oracle.layout import sf_to_storage
from w4a4_rank_absorbed_b200.synth import make_workload, small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _assert_bytes(gpu: torch.Tensor, ref: np.ndarray, what: str):
    a = u8_host(gpu)
    b = np.asarray(ref, dtype=np.uint8).reshape(-1)
    assert a.size == b.size, f"{what}: size {a.size} vs {b.size}"
    assert np.array_equal(a, b), f"{what}: " + mismatch_report(a, b)


@pytest.mark.parametrize("K,N,r", [(512, 512, 32), (256, 144, 16), (1024, 400, 0), (320, 256, 48),
                                   (64, 16, 16), (768, 1040, 128)])
def test_pack_weight_bitexact(K, N, r):
    wl = small_case(32, K, N, r, seed=K + N + r)
    dec = oracle_layer(wl, r)
    g = GpuLayer(dec, wl.bias)
    pw = OL.pack_weight(dec.R32)
    assert g.gs_w == pw.gs_w
    ref = oracle_storage(pw=pw)
    _assert_bytes(g.Wq, ref["Wq"], "Wq")
    _assert_bytes(g.SFw, ref["SFw"], "SFw")
    if r:
        assert np.array_equal(bf16_host(g.L2p), dec.L2b.T)
    g.check_errors()


@pytest.mark.parametrize("M,K,r", [(256, 512, 32), (100, 512, 32), (37, 256, 16), (300, 1024, 64), (64, 512, 0),
                                   (130, 512, 48), (64, 256, 80), (64, 256, 128), (1, 64, 16), (160, 192, 96),
                                   (33, 320, 112)])
def test_quantize_act_bitexact(M, K, r):
    wl = small_case(M, K, 128, r, seed=M * 7 + K + r)
    dec = oracle_layer(wl, r)
    assert dec.L1f.shape[1] == r       # N >= r, so the rank is not clamped
    g = GpuLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(wl.X))
    qa = OL.quantize_act(wl.X, dec.inv_s, dec.gs_x, dec.L1f)
    ref = oracle_storage(qa=qa)
    _assert_bytes(Xq, ref["Xq"], "Xq")
    _assert_bytes(SFx, ref["SFx"], "SFx")
    if r:
        check_las(LAs, wl.X, dec.L1f, g.lr_scale)
    g.check_errors()


def _oracle_inputs_to_device(qa, pw, dec, lr_scale, r_expected):
    """The oracle's codes/scales and a hi/lo split of its float64 low-rank product (in the LAs layout:
    interleaved by 16 columns), as device buffers.

    The buffers are sized by the decomposition's rank, which the launch must use: a kernel
    told a larger r would read past LAs and L2p.
    """
    assert dec.L1f.shape[1] == r_expected, f"decomposition rank {dec.L1f.shape[1]} != {r_expected}"
    Xq = torch.from_numpy(OC.pack_codes(qa.codes)).cuda()
    SFx = torch.from_numpy(sf_to_storage(qa.scales)).cuda()
    Wq = torch.from_numpy(OC.pack_codes(pw.codes)).cuda()
    SFw = torch.from_numpy(sf_to_storage(pw.scales)).cuda()
    r = dec.L1f.shape[1]
    if r:
        v = torch.from_numpy((qa.LA * np.float64(lr_scale)).astype(np.float32))
        hi = v.to(torch.bfloat16)
        lo = (v - hi.float()).to(torch.bfloat16)
        LAs = bf16_dev(las_join(hi.double().numpy(), lo.double().numpy()))
        L2p = bf16_dev(np.ascontiguousarray(dec.L2b.T))
    else:
        LAs = L2p = None
    return Xq, SFx, Wq, SFw, LAs, L2p


@pytest.mark.parametrize("y_fp32", [False, True])
@pytest.mark.parametrize("M,N,K,r,use_bias", [(256, 512, 512, 32, True), (200, 400, 320, 16, True),
                                              (128, 256, 64, 0, False), (384, 768, 1024, 32, True),
                                              (70, 144, 256, 64, False), (129, 272, 576, 48, True),
                                              (1, 16, 64, 16, True), (520, 1296, 1536, 128, True),
                                              (128, 128, 128, 0, True), (256, 256, 128, 16, False),
                                              (128, 256, 64, 16, True)])
def test_linear_on_oracle_codes(M, N, K, r, use_bias, y_fp32):
    from w4a4_rank_absorbed_b200 import svdq as C
    wl = small_case(M, K, N, r, seed=M + 3 * N + K)
    dec = oracle_layer(wl, r)
    pw = OL.pack_weight(dec.R32)
    qa = OL.quantize_act(wl.X, dec.inv_s, dec.gs_x, dec.L1f)
    gs_x, gs_w = np.float32(dec.gs_x), pw.gs_w
    lr_scale = np.float32(1.0 / (np.float64(gs_x) * np.float64(gs_w)))
    Xq, SFx, Wq, SFw, LAs, L2p = _oracle_inputs_to_device(qa, pw, dec, lr_scale, r)
    bias = bf16_dev(wl.bias) if use_bias else None
    Y = torch.empty((M, N), dtype=torch.float32 if y_fp32 else torch.bfloat16, device="cuda")
    C.svdq_linear(Xq, SFx, float(gs_x), Wq, SFw, float(gs_w), LAs, L2p, r, bias, Y, int(y_fp32), M, N, K)
    torch.cuda.synchronize()
    Y_or = OL.linear(qa, gs_x, pw, dec.L2b, wl.bias if use_bias else None)
    check_y(Y.float().cpu().numpy().astype(np.float64), Y_or, bf16=not y_fp32, what=f"Y {M}x{N}x{K} r={r}")
    st, site = C.svdq_get_device_error()
    assert st == 0, site


@pytest.mark.parametrize("M,N,K,r", [(256, 512, 512, 32), (300, 528, 768, 16), (64, 256, 256, 0),
                                     (129, 400, 320, 64)])
def test_layer_end_to_end(M, N, K, r):
    wl = small_case(M, K, N, r, seed=11 + M + N)
    dec = oracle_layer(wl, r)
    g = GpuLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(wl.X))
    Y16 = g.linear(Xq, SFx, LAs)
    Y32 = g.linear(Xq, SFx, LAs, y_fp32=True)
    torch.cuda.synchronize()
    Y_or, qa, pw = OL.svdq_reference(wl.X, dec.inv_s, dec.gs_x, dec.L1f, dec.L2b, dec.R32, wl.bias)
    ref = oracle_storage(qa, pw)
    _assert_bytes(Xq, ref["Xq"], "Xq")
    _assert_bytes(g.Wq, ref["Wq"], "Wq")
    check_y(Y16.float().cpu().numpy().astype(np.float64), Y_or, bf16=True, what="bf16 Y")
    check_y(Y32.cpu().numpy().astype(np.float64), Y_or, bf16=False, what="fp32 Y")
    g.check_errors()


def test_tiny_config_and_method_effect():
    wl = make_workload("tiny")
    dec = oracle_layer(wl)
    g = GpuLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(wl.X))
    Y = g.linear(Xq, SFx, LAs, y_fp32=True).cpu().numpy().astype(np.float64)
    Y_or, _, _ = OL.svdq_reference(wl.X, dec.inv_s, dec.gs_x, dec.L1f, dec.L2b, dec.R32, wl.bias)
    check_y(Y, Y_or, bf16=False, what="tiny")
    exact = wl.X @ wl.W + wl.bias[None, :]
    assert OL.rel_fro(Y, exact) < OL.rel_fro(OL.w4a4_plain(wl.X, wl.W, wl.bias), exact)
    g.check_errors()


def test_edge_values():
    # all-zero rows and groups, negative zeros, values at E2M1 ties, and a calibration scale that makes
    # some runtime groups saturate their UE4M3 scale (gs_x calibrated on smaller activations), others
    # fall to subnormal scales or to a zero scale.
    M, K, N, r = 96, 256, 64, 16
    wl = small_case(M, K, N, r, seed=123)
    X = wl.X.copy()
    X[5] = 0.0
    X[7, 16:48] = 0.0
    X[9, :16] = -0.0
    X[11, :16] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0,
                           -6.0])
    X[13, :] *= 1e4
    X[15, :] *= 1e-4            # block scales in the UE4M3 subnormal range
    X[17, :] *= 1e-7            # block scales that round to 0: all codes 0
    dec = OD.decompose(X, wl.W, r, 0.5, X_cal=wl.X)     # calibrated without the scaled rows
    X = np.asarray(torch.from_numpy(X).to(torch.bfloat16).double().numpy())
    g = GpuLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(X))
    qa = OL.quantize_act(X, dec.inv_s, dec.gs_x, dec.L1f)
    ref = oracle_storage(qa=qa)
    assert (qa.scales[13] == 0x7E).any(), "expected saturating scales in row 13"
    assert ((qa.scales[15] > 0) & (qa.scales[15] < 8)).any(), "expected subnormal scales in row 15"
    assert (qa.scales[17] == 0).all(), "expected zero scales in row 17"
    _assert_bytes(Xq, ref["Xq"], "Xq")
    _assert_bytes(SFx, ref["SFx"], "SFx")
    check_las(LAs, X, dec.L1f, g.lr_scale)
    g.check_errors()


def test_bounded_wait_reports_timeout_and_context_survives():
    from w4a4_rank_absorbed_b200 import svdq as C
    wl = small_case(128, 256, 256, 16, seed=3)
    dec = oracle_layer(wl, 16)
    g = GpuLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(wl.X))
    Y = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
    C.svdq_linear_debug(Xq, SFx, float(g.gs_x), g.Wq, g.SFw, float(g.gs_w), LAs, g.L2p, 16, g.bias, Y, 0,
                        128, 256, 256, 1, 2_000_000)
    st, site = C.svdq_get_device_error()
    assert st == C.SVDQ_ERR_TIMEOUT and site != 0
    # the context is still usable and the error word was cleared
    Y2 = g.linear(Xq, SFx, LAs)
    torch.cuda.synchronize()
    assert C.svdq_get_device_error()[0] == 0
    Y_or, _, _ = OL.svdq_reference(wl.X, dec.inv_s, dec.gs_x, dec.L1f, dec.L2b, dec.R32, wl.bias)
    check_y(Y2.float().cpu().numpy().astype(np.float64), Y_or, bf16=True)


def test_repeated_launches_are_identical_and_error_free():
    # Pipelines with many barriers in flight: repeat the forward and require bit-identical results
    # and a clean device error word (catches ordering races that a single launch may miss).
    M, K, N, r = 1152, 3072, 1536, 32
    wl = small_case(M, K, N, r, seed=77)
    dec = oracle_layer(wl, r)
    g = GpuLayer(dec, wl.bias)
    X = bf16_dev(wl.X)
    ref = None
    for _ in range(40):
        Xq, SFx, LAs = g.quantize(X)
        Y = g.linear(Xq, SFx, LAs)
        torch.cuda.synchronize()
        cur = (Xq.cpu().numpy().tobytes(), SFx.cpu().numpy().tobytes(), LAs.view(torch.int16).cpu().numpy().tobytes(),
               Y.view(torch.int16).cpu().numpy().tobytes())
        if ref is None:
            ref = cur
        else:
            assert cur == ref
    g.check_errors()


@pytest.mark.parametrize("M,K,r", [(256, 512, 32), (300, 1024, 64), (1152, 3072, 32), (37, 256, 16), (130, 512, 48)])
def test_lowrank_down_equals_the_fused_down_projection(M, K, r):
    # The separate down-projection (unfused pipeline) runs the fused kernel's MMA path without the
    # quantization: its LAs must be bit-identical to the fused kernel's, and within the LA bound of the
    # oracle's float64 product.
    from w4a4_rank_absorbed_b200 import svdq as C
    wl = small_case(M, K, 128, r, seed=3 * M + K + r)
    dec = oracle_layer(wl, r)
    assert dec.L1f.shape[1] == r, "the buffers are sized by the decomposition's rank"
    g = GpuLayer(dec, wl.bias)
    X = bf16_dev(wl.X)
    _, _, LAs_fused = g.quantize(X)
    LAs = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda")
    C.svdq_lowrank_down(X, M, K, g.L1fT, r, float(g.lr_scale), LAs, C.new_workspace(M, K, r))
    torch.cuda.synchronize()
    assert torch.equal(LAs.view(torch.int16), LAs_fused.view(torch.int16))
    check_las(LAs, wl.X, dec.L1f, g.lr_scale)
    g.check_errors()


@pytest.mark.parametrize("M,N,K,r", [(256, 512, 512, 32), (300, 528, 768, 16), (129, 400, 320, 64),
                                     (520, 1296, 1536, 128)])
def test_unfused_pipeline_matches_oracle(M, N, K, r):
    # In-house unfused form of the layer: quantize without the branch, a separate down-projection that
    # re-reads X, the plain NVFP4 GEMM, a separate up-projection that reads and rewrites Y.  In fp32
    # output the literal gate applies.
    from w4a4_rank_absorbed_b200 import svdq as C
    wl = small_case(M, K, N, r, seed=19 + M + N + r)
    dec = oracle_layer(wl, r)
    g = GpuLayer(dec, wl.bias)
    X = bf16_dev(wl.X)
    Xq = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    SFx = torch.empty(C.svdq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
    C.svdq_quantize_act(X, M, K, g.inv_s, float(g.gs_x), None, 0, 1.0, Xq, SFx, None)
    LA = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda")
    C.svdq_lowrank_down(X, M, K, g.L1fT, r, 1.0, LA, C.new_workspace(M, K, r))
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    C.svdq_linear(Xq, SFx, float(g.gs_x), g.Wq, g.SFw, float(g.gs_w), None, None, 0, g.bias, Y, 1, M, N, K)
    C.svdq_lowrank_up(LA, g.L2p, r, 1.0, Y, 1, M, N)
    torch.cuda.synchronize()
    g.check_errors()
    Y_or, qa, _ = OL.svdq_reference(wl.X, dec.inv_s, dec.gs_x, dec.L1f, dec.L2b, dec.R32, wl.bias)
    _assert_bytes(Xq, oracle_storage(qa=qa)["Xq"], "Xq")
    check_y(Y.cpu().numpy().astype(np.float64), Y_or, bf16=False, what=f"unfused {M}x{N}x{K} r={r}")


def test_workspace_is_reusable_and_left_clean():
    # The ticket words of the workspace return to 0 after every call, so one zeroed workspace serves
    # any number of calls (and shapes no larger than it was sized for); results repeat bit for bit.
    from w4a4_rank_absorbed_b200 import svdq as C
    M, K, r = 640, 2048, 32
    wl = small_case(M, K, 64, r, seed=99)
    dec = oracle_layer(wl, r)
    g = GpuLayer(dec, wl.bias)
    ws = C.new_workspace(M, K, r)
    X = bf16_dev(wl.X)
    outs = []
    for _ in range(3):
        Xq = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        SFx = torch.empty(C.svdq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
        LAs = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda")
        C.svdq_quantize_act(X, M, K, g.inv_s, float(g.gs_x), g.L1fT, r, float(g.lr_scale), Xq, SFx, LAs, ws)
        torch.cuda.synchronize()
        outs.append((Xq.cpu(), SFx.cpu(), LAs.view(torch.int16).cpu()))
        tickets = ws[:256].cpu()
        assert int(tickets.sum()) == 0
    for o in outs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(o, outs[0]))
    check_las(outs[0][2].view(torch.bfloat16), wl.X, dec.L1f, g.lr_scale)
    g.check_errors()
