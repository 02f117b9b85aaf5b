"""Parity at the full workload sizes, in the launch configuration the benchmark times.

Every byte of the packed weight and of the quantized activations is compared
with the oracle, the low-rank product on every row, and the layer output on
every element, once with bf16 output and once with fp32 output (the oracle
does a FLUX-sized layer in a few seconds).
"""
import numpy as np
import pytest
import torch

from helpers import (GpuLayer, OC, OD, OL, bf16_dev, check_las, check_y, mismatch_report,
                     oracle_storage, require_gpu, u8_host)
from oracle import mlp as OM
from w4a4_rank_absorbed_b200.synth import make_workload

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check_layer(wl, dec, X, what):
    g = GpuLayer(dec, wl.bias)
    M, K = X.shape
    Xq, SFx, LAs = g.quantize(bf16_dev(X))
    Y16 = g.linear(Xq, SFx, LAs)
    Y32 = g.linear(Xq, SFx, LAs, y_fp32=True)
    torch.cuda.synchronize()
    g.check_errors()
    pw = OL.pack_weight(dec.R32)
    qa = OL.quantize_act(X, dec.inv_s, dec.gs_x, dec.L1f)
    assert g.gs_w == pw.gs_w
    ref = oracle_storage(qa=qa, pw=pw)
    for name, buf in (("Wq", g.Wq), ("SFw", g.SFw), ("Xq", Xq), ("SFx", SFx)):
        a, b = u8_host(buf), ref[name]
        assert np.array_equal(a, b), f"{what} {name}: " + mismatch_report(a, b)
    if dec.L1f.shape[1]:
        check_las(LAs.cpu(), X, dec.L1f, g.lr_scale)
    Y_or = OL.linear(qa, dec.gs_x, pw, dec.L2b, wl.bias)
    rel16, mx16 = check_y(Y16.float().cpu().numpy().astype(np.float64), Y_or, bf16=True, what=what + " bf16")
    rel32, mx32 = check_y(Y32.cpu().numpy().astype(np.float64), Y_or, bf16=False, what=what + " fp32")
    print(f"{what}: bf16 rel-Fro {rel16:.3e} max/rms {mx16:.3e}; fp32 rel-Fro {rel32:.3e} max/rms {mx32:.3e}")
    return g, Y_or


def test_qkv_projection():
    wl = make_workload("qkv")
    dec = OD.decompose(wl.X, wl.W, wl.r, wl.alpha)
    _check_layer(wl, dec, wl.X, "qkv")


def test_large_batch():
    wl = make_workload("large")
    dec = OD.decompose(wl.X, wl.W, wl.r, wl.alpha)
    _check_layer(wl, dec, wl.X, "large")


def test_mlp_pair_fc1_gelu_fc2():
    wl1 = make_workload("fc1")
    dec1 = OD.decompose(wl1.X, wl1.W, wl1.r, wl1.alpha)
    _, Y1_or = _check_layer(wl1, dec1, wl1.X, "fc1")
    # fc2's input is the oracle's GELU of the oracle's fc1 output (bf16 in, bf16 out); fc2 is
    # calibrated on it and both sides run fc2 on it
    X2 = OM.gelu_bf16(OD.bf16_round(Y1_or))
    wl2 = make_workload("fc2")
    wl2.X = X2
    dec2 = OD.decompose(X2, wl2.W, wl2.r, wl2.alpha)
    _check_layer(wl2, dec2, X2, "fc2")


@pytest.mark.parametrize("lora", [False, True])
def test_rank_sweep(lora):
    for r in (16, 32, 64):
        wl = make_workload(f"sweep_r{r}" + ("_lora" if lora else ""))
        dec = OD.decompose(wl.X, wl.W, r, wl.alpha, wl.lora_A, wl.lora_B)
        assert dec.L1f.shape[1] == r + (16 if lora else 0)
        _check_layer(wl, dec, wl.X, f"sweep r={r} lora={lora}")
