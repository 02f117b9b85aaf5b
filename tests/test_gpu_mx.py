"""Parity of the MXFP4 form of the layer (blocks of 32, E8M0 scales, no global scale) against the oracle.

Codes and scales must match the oracle's MXFP4 codec byte for byte; the output is held to the same
gate as the NVFP4 layer (rel-Frobenius and max-abs against the unrounded float64 oracle)."""
import numpy as np
import pytest
import torch

from helpers import (bf16_dev, bf16_host, check_las, check_y, f32_dev, las_join, mismatch_report, oracle_layer,
                     require_gpu, u8_host)
from oracle import codec as OC
from oracle import mx as OM
from oracle.layout import sf_to_storage
from w4a4_rank_absorbed_b200.synth import small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _C():
    from w4a4_rank_absorbed_b200 import svdq as C
    return C


def _assert_bytes(gpu: torch.Tensor, ref: np.ndarray, what: str):
    a = u8_host(gpu)
    b = np.asarray(ref, dtype=np.uint8).reshape(-1)
    assert a.size == b.size, f"{what}: size {a.size} vs {b.size}"
    assert np.array_equal(a, b), f"{what}: " + mismatch_report(a, b)


class MxLayer:
    """pack -> quantize -> linear of the MXFP4 entry points on oracle-decomposed data."""

    def __init__(self, dec, bias):
        C = _C()
        K, N = dec.R32.shape
        r = dec.L1f.shape[1]
        self.K, self.N, self.r = K, N, r
        self.R = f32_dev(dec.R32)
        self.L2b = bf16_dev(dec.L2b) if r else None
        self.Wq = torch.full((N, K // 2), 0x5A, dtype=torch.uint8, device="cuda")
        self.SFw = torch.full((C.svdq_mx_sf_bytes(N, K),), 0xAB, dtype=torch.uint8, device="cuda")
        self.L2p = torch.empty((N, r), dtype=torch.bfloat16, device="cuda") if r else None
        C.svdq_pack_weight_mx(self.R, self.L2b, K, N, r, self.Wq, self.SFw, self.L2p)
        self.inv_s = f32_dev(dec.inv_s)
        self.L1fT = bf16_dev(np.ascontiguousarray(dec.L1f.T)) if r else None
        self.bias = bf16_dev(bias) if bias is not None else None
        self.ws = {}

    def quantize(self, X_dev):
        C = _C()
        M = X_dev.shape[0]
        Xq = torch.full((M, self.K // 2), 0x5A, dtype=torch.uint8, device="cuda")
        SFx = torch.full((C.svdq_mx_sf_bytes(M, self.K),), 0xAB, dtype=torch.uint8, device="cuda")
        LAs = torch.empty((M, 2 * self.r), dtype=torch.bfloat16, device="cuda") if self.r else None
        if M not in self.ws:
            self.ws[M] = C.new_workspace(M, self.K, self.r)
        C.svdq_quantize_act_mx(X_dev, M, self.K, self.inv_s, self.L1fT, self.r, 1.0, Xq, SFx, LAs, self.ws[M])
        return Xq, SFx, LAs

    def linear(self, Xq, SFx, LAs, y_fp32=False, bias=True):
        M = Xq.shape[0]
        Y = torch.empty((M, self.N), dtype=torch.float32 if y_fp32 else torch.bfloat16, device="cuda")
        _C().svdq_linear_mx(Xq, SFx, self.Wq, self.SFw, LAs, self.L2p, self.r, self.bias if bias else None, Y,
                            1 if y_fp32 else 0, M, self.N, self.K)
        return Y


def _check_errors():
    st, site = _C().svdq_get_device_error()
    assert st == 0, f"device error {st} at site {site:#x}"


def test_mx_sf_bytes_and_shape_rules():
    C = _C()
    assert C.svdq_mx_sf_bytes(1, 128) == 128 * 4
    assert C.svdq_mx_sf_bytes(129, 384) == 256 * 12
    assert C.svdq_mx_sf_bytes(16, 64) == 0          # K % 128 != 0
    X = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    inv_s = torch.ones(64, dtype=torch.float32, device="cuda")
    Xq = torch.zeros((16, 32), dtype=torch.uint8, device="cuda")
    SFx = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(C.SVDQError) as e:
        C.svdq_quantize_act_mx(X, 16, 64, inv_s, None, 0, 1.0, Xq, SFx, None)
    assert e.value.status == C.SVDQ_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("K,N,r", [(512, 512, 32), (256, 144, 16), (1024, 400, 0), (384, 256, 48),
                                   (128, 16, 16), (768, 1040, 128)])
def test_pack_weight_mx_bitexact(K, N, r):
    wl = small_case(32, K, N, r, seed=5 * K + N + r)
    dec = oracle_layer(wl, r)
    g = MxLayer(dec, wl.bias)
    torch.cuda.synchronize()
    pw = OM.mx_pack_weight(dec.R32)
    _assert_bytes(g.Wq, OC.pack_codes(pw.codes), "Wq")
    _assert_bytes(g.SFw, sf_to_storage(pw.scales), "SFw")
    if r:
        assert np.array_equal(bf16_host(g.L2p), dec.L2b.T)
    _check_errors()


@pytest.mark.parametrize("M,K,r", [(256, 512, 32), (100, 512, 32), (37, 256, 16), (300, 1024, 64), (64, 512, 0),
                                   (130, 384, 48), (1, 128, 16), (33, 640, 112), (160, 128, 96)])
def test_quantize_act_mx_bitexact(M, K, r):
    wl = small_case(M, K, 128, r, seed=M * 3 + K + r)
    dec = oracle_layer(wl, r)
    assert dec.L1f.shape[1] == r
    g = MxLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(wl.X))
    torch.cuda.synchronize()
    qa = OM.mx_quantize_act(wl.X, dec.inv_s, dec.L1f)
    _assert_bytes(Xq, OC.pack_codes(qa.codes), "Xq")
    _assert_bytes(SFx, sf_to_storage(qa.scales), "SFx")
    if r:
        check_las(LAs, wl.X, dec.L1f, 1.0)
    _check_errors()


def _mx_oracle_to_device(qa, pw, dec):
    Xq = torch.from_numpy(OC.pack_codes(qa.codes)).cuda()
    SFx = torch.from_numpy(sf_to_storage(qa.scales)).cuda()
    Wq = torch.from_numpy(OC.pack_codes(pw.codes)).cuda()
    SFw = torch.from_numpy(sf_to_storage(pw.scales)).cuda()
    r = dec.L1f.shape[1]
    if r:
        v = torch.from_numpy(qa.LA.astype(np.float32))
        hi = v.to(torch.bfloat16)
        lo = (v - hi.float()).to(torch.bfloat16)
        LAs = bf16_dev(las_join(hi.double().numpy(), lo.double().numpy()))
        L2p = bf16_dev(np.ascontiguousarray(dec.L2b.T))
    else:
        LAs = L2p = None
    return Xq, SFx, Wq, SFw, LAs, L2p


@pytest.mark.parametrize("y_fp32", [False, True])
@pytest.mark.parametrize("M,N,K,r,use_bias", [(256, 512, 512, 32, True), (200, 400, 384, 16, True),
                                              (128, 256, 128, 0, False), (384, 768, 1024, 32, True),
                                              (70, 144, 256, 64, False), (129, 272, 640, 48, True),
                                              (1, 16, 128, 16, True), (520, 1296, 1536, 128, True)])
def test_linear_mx_on_oracle_codes(M, N, K, r, use_bias, y_fp32):
    C = _C()
    wl = small_case(M, K, N, r, seed=2 * M + N + K)
    dec = oracle_layer(wl, r)
    assert dec.L1f.shape[1] == r
    pw = OM.mx_pack_weight(dec.R32)
    qa = OM.mx_quantize_act(wl.X, dec.inv_s, dec.L1f)
    Xq, SFx, Wq, SFw, LAs, L2p = _mx_oracle_to_device(qa, pw, dec)
    bias = bf16_dev(wl.bias) if use_bias else None
    Y = torch.empty((M, N), dtype=torch.float32 if y_fp32 else torch.bfloat16, device="cuda")
    C.svdq_linear_mx(Xq, SFx, Wq, SFw, LAs, L2p, r, bias, Y, int(y_fp32), M, N, K)
    torch.cuda.synchronize()
    Y_or = OM.mx_linear(qa, pw, dec.L2b, wl.bias if use_bias else None)
    check_y(Y.float().cpu().numpy().astype(np.float64), Y_or, bf16=not y_fp32, what=f"MX Y {M}x{N}x{K} r={r}")
    _check_errors()


@pytest.mark.parametrize("M,N,K,r", [(256, 512, 512, 32), (300, 528, 768, 16), (64, 256, 256, 0),
                                     (129, 400, 384, 64), (1024, 3072, 3072, 32)])
def test_mx_layer_end_to_end(M, N, K, r):
    wl = small_case(M, K, N, r, seed=17 + M + N)
    dec = oracle_layer(wl, r)
    g = MxLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(wl.X))
    Y16 = g.linear(Xq, SFx, LAs)
    Y32 = g.linear(Xq, SFx, LAs, y_fp32=True)
    torch.cuda.synchronize()
    Y_or, qa, pw = OM.mx_reference(wl.X, dec.inv_s, dec.L1f, dec.L2b, dec.R32, wl.bias)
    _assert_bytes(Xq, OC.pack_codes(qa.codes), "Xq")
    _assert_bytes(SFx, sf_to_storage(qa.scales), "SFx")
    _assert_bytes(g.Wq, OC.pack_codes(pw.codes), "Wq")
    check_y(Y16.float().cpu().numpy().astype(np.float64), Y_or, bf16=True, what="MX bf16 Y")
    check_y(Y32.cpu().numpy().astype(np.float64), Y_or, bf16=False, what="MX fp32 Y")
    _check_errors()


def test_mx_edge_values():
    """Zero blocks, values that saturate (6 < |x| * 2^-X < 8 cannot occur for the block maximum, but
    the block max itself sits at every binade edge), tiny and huge magnitudes that reach the E8M0 clamp."""
    M, K, N, r = 128, 512, 128, 16
    wl = small_case(M, K, N, r, seed=99)
    dec = oracle_layer(wl, r)
    X = wl.X.copy()
    X[3, :] = 0.0                                   # a zero row: every block of it is zero
    X[5, 32:64] = 0.0                               # one zero block
    X[7, :32] = 2.0 ** -133                         # bf16 subnormal: scale clamps at 2^-127
    X[9, 64:96] = 2.0 ** 100                        # large, but still far from bf16 overflow
    X[11, 128:160] = np.where(np.arange(32) % 2, 7.0, -8.0)   # the maximum on a binade edge
    X[13, 160:192] = 6.0 * 2.0 ** np.arange(-16, 16)          # every binade within one block
    inv_s = np.ones_like(dec.inv_s)
    dec.inv_s = inv_s
    g = MxLayer(dec, wl.bias)
    Xq, SFx, LAs = g.quantize(bf16_dev(X))
    torch.cuda.synchronize()
    qa = OM.mx_quantize_act(X, inv_s, dec.L1f)
    _assert_bytes(Xq, OC.pack_codes(qa.codes), "Xq")
    _assert_bytes(SFx, sf_to_storage(qa.scales), "SFx")
    sc = qa.scales
    assert sc[3].max() == 0 and sc[5, 1] == 0 and sc[7, 0] == 0
    _check_errors()
