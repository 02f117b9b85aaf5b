"""Shared helpers of the GPU parity tests: run the CUDA path on oracle-decomposed inputs and compare."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import codec as OC
from oracle import decompose as OD
from oracle import linear as OL
from oracle.layout import sf_to_storage

# Tolerances of the layer output against the float64 oracle (the stated output tolerances):
REL_FRO = 2e-3          # ||Y - Y_or||_F / ||Y_or||_F
MAX_ABS_RMS = 1e-2      # max |Y - Y_or| <= 1e-2 rms(Y_or)   (+ half a bf16 ulp of Y_or for bf16 output)
LA_REL = 2e-5           # |LAs_hi + LAs_lo - lr_scale X L1f| <= 2e-5 lr_scale (|X| |L1f|)
REL_ROUNDED_MARGIN = 1e-4   # bf16 output: rel-Frobenius may exceed the rounded oracle's own by this much


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.fail(f"needs compute capability 10.0, found {major}.{minor}")
    from w4a4_rank_absorbed_b200 import build, svdq
    build.build()
    svdq.load_library()


def bf16_dev(a) -> torch.Tensor:
    """float64 values that are exactly bf16 -> bf16 device tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    assert np.array_equal(t.float().numpy().astype(np.float64), np.asarray(a, dtype=np.float64)), "not bf16-exact"
    return t.cuda()


def f32_dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def u8_host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().astype(np.uint8).reshape(-1)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def bf16_bits(a) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def half_ulp_bf16(y: np.ndarray) -> np.ndarray:
    a = np.abs(y)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)        # half of the bf16 spacing 2^(e-7)


def check_y(Y_gpu: np.ndarray, Y_or: np.ndarray, bf16: bool, what: str = ""):
    """Output gate against the unrounded float64 oracle.

    rel-Frobenius ||Y - Y_or||_F / ||Y_or||_F <= 2e-3 in both output modes (the bf16 rounding of the
    output alone costs about 1.7e-3 of it, which is why the low-rank branch is carried as a hi/lo pair).
    max-abs: fp32 output <= 1e-2 rms(Y_or); bf16 output <= 1e-2 rms(Y_or) + half a bf16 ulp of Y_or,
    since rounding a value near 4 sigma to bf16 alone moves it by up to 1.6e-2 rms."""
    d = np.abs(Y_gpu - Y_or)
    rms = float(np.sqrt(np.mean(Y_or ** 2)))
    rel = float(np.linalg.norm(Y_gpu - Y_or) / np.linalg.norm(Y_or))
    rel_bound = REL_FRO
    if bf16:
        # The best any bf16 output can do is the correctly rounded oracle; on outputs of a few dozen
        # elements its own rel-Frobenius can exceed 2e-3 (2.05e-3 on a 1 x 16 output), so the bound
        # is never below that figure plus a small margin for the float32 arithmetic.
        rho = float(np.linalg.norm(OD.bf16_round(Y_or) - Y_or) / np.linalg.norm(Y_or))
        rel_bound = max(REL_FRO, rho + REL_ROUNDED_MARGIN)
    bound = MAX_ABS_RMS * rms + (half_ulp_bf16(Y_or) if bf16 else 0.0)
    worst = float(np.max(d - bound))
    assert rel <= rel_bound, f"{what} rel-Frobenius {rel:.3e} > {rel_bound:.3e}"
    assert worst <= 0, f"{what} max-abs error exceeds bound by {worst:.3e} (rms {rms:.3e})"
    return rel, float(d.max() / rms)


def oracle_layer(wl, r=None, X_cal=None):
    r = wl.r if r is None else r
    return OD.decompose(wl.X, wl.W, r, wl.alpha, wl.lora_A, wl.lora_B, X_cal=X_cal)


class GpuLayer:
    """Runs pack -> quantize -> linear through the C ABI on oracle-decomposed data."""

    def __init__(self, dec, bias):
        from w4a4_rank_absorbed_b200 import svdq as C
        self.C = C
        K, N = dec.R32.shape
        r = dec.L1f.shape[1]
        self.K, self.N, self.r = K, N, r
        self.dec = dec
        self.R = f32_dev(dec.R32)
        self.L2b = bf16_dev(dec.L2b) if r else None
        self.Wq = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        self.SFw = torch.full((C.svdq_sf_bytes(N, K),), 0xAB, dtype=torch.uint8, device="cuda")
        self.gs_w_dev = torch.empty(1, dtype=torch.float32, device="cuda")
        self.L2p = torch.empty((N, r), dtype=torch.bfloat16, device="cuda") if r else None
        self.gs_w = np.float32(C.svdq_pack_weight(self.R, self.L2b, K, N, r, self.Wq, self.SFw, self.gs_w_dev,
                                                  self.L2p))
        assert self.gs_w == np.float32(self.gs_w_dev.item())
        self.gs_x = np.float32(dec.gs_x)
        self.lr_scale = np.float32(1.0 / (np.float64(self.gs_x) * np.float64(self.gs_w)))
        self.inv_s = f32_dev(dec.inv_s)
        self.L1fT = bf16_dev(np.ascontiguousarray(dec.L1f.T)) if r else None
        self.bias = bf16_dev(bias) if bias is not None else None
        self.ws = {}

    def quantize(self, X_dev):
        C = self.C
        M = X_dev.shape[0]
        Xq = torch.empty((M, self.K // 2), dtype=torch.uint8, device="cuda")
        SFx = torch.full((C.svdq_sf_bytes(M, self.K),), 0xAB, dtype=torch.uint8, device="cuda")
        LAs = torch.empty((M, 2 * self.r), dtype=torch.bfloat16, device="cuda") if self.r else None
        if M not in self.ws:
            self.ws[M] = C.new_workspace(M, self.K, self.r)
        C.svdq_quantize_act(X_dev, M, self.K, self.inv_s, float(self.gs_x), self.L1fT, self.r,
                            float(self.lr_scale), Xq, SFx, LAs, self.ws[M])
        return Xq, SFx, LAs

    def linear(self, Xq, SFx, LAs, y_fp32=False, bias=True):
        M = Xq.shape[0]
        Y = torch.empty((M, self.N), dtype=torch.float32 if y_fp32 else torch.bfloat16, device="cuda")
        self.C.svdq_linear(Xq, SFx, float(self.gs_x), self.Wq, self.SFw, float(self.gs_w), LAs, self.L2p,
                           self.r, self.bias if bias else None, Y, 1 if y_fp32 else 0, M, self.N, self.K)
        return Y

    def check_errors(self):
        st, site = self.C.svdq_get_device_error()
        assert st == 0, f"device error {st} at site {site:#x}"


def la_bound(X, L1f, lr_scale):
    return LA_REL * float(lr_scale) * (np.abs(X) @ np.abs(L1f))


def las_split(las: np.ndarray, r: int):
    """(hi, lo) of an LAs buffer (M x 2r, hi and lo interleaved by 16 columns)."""
    g = las.reshape(las.shape[0], r // 16, 2, 16)
    return g[:, :, 0, :].reshape(-1, r), g[:, :, 1, :].reshape(-1, r)


def las_join(hi: np.ndarray, lo: np.ndarray) -> np.ndarray:
    """The LAs layout from its hi and lo halves (M x r each): interleaved by 16 columns."""
    M, r = hi.shape
    return np.stack([hi.reshape(M, r // 16, 16), lo.reshape(M, r // 16, 16)], axis=2).reshape(M, 2 * r)


def check_las(LAs_gpu: torch.Tensor, X, L1f, lr_scale, rows=None):
    r = L1f.shape[1]
    las = bf16_host(LAs_gpu)
    hi, lo = las_split(las, r)
    v = hi + lo
    Xs = X if rows is None else X[rows]
    if rows is not None:
        v = v[rows]
    ref = (Xs @ L1f) * np.float64(lr_scale)
    err = np.abs(v - ref)
    bound = la_bound(Xs, L1f, lr_scale) + 1e-30
    assert np.all(err <= bound), f"LAs error {float(np.max(err / bound)):.3f} of bound"
    # hi is the bf16 rounding of v: |lo| <= half an ulp of hi
    assert np.all(np.abs(lo) <= half_ulp_bf16(hi) * 1.0000001 + 1e-38)


def oracle_storage(qa=None, pw=None):
    out = {}
    if qa is not None:
        out["Xq"] = OC.pack_codes(qa.codes).reshape(-1)
        out["SFx"] = sf_to_storage(qa.scales)
    if pw is not None:
        out["Wq"] = OC.pack_codes(pw.codes).reshape(-1)
        out["SFw"] = sf_to_storage(pw.scales)
    return out


def mismatch_report(a: np.ndarray, b: np.ndarray) -> str:
    bad = np.nonzero(a != b)[0]
    return f"{bad.size} of {a.size} bytes differ; first at {bad[:8].tolist()}: gpu {a[bad[:8]].tolist()} " \
           f"oracle {b[bad[:8]].tolist()}"


__all__ = ["OC", "OD", "OL"]
