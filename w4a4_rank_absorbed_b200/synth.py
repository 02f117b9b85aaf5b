"""Seeded synthetic workloads for the SVDQuant linear layer.

This module only draws random numbers. It holds none of the method's
arithmetic (no smoothing, no SVD, no quantization), so that both the CUDA
path and the CPU oracle can take their inputs from it without sharing any
of the computation they are compared on.

The workloads follow the shapes and value distributions of the diffusion
transformer layers that the SVDQuant pages discuss (FLUX.1 attention QKV
projection and MLP, "SVDQuant: Absorbing Outliers by Low-Rank Components
for 4-Bit Diffusion Models", abstract; "From SmoothQuant to SVDQuant",
section "SVDQuant (W4A4)"): activations with a few outlier channels (the
pages observe that activation outliers sit in a few fixed channels,
"From SmoothQuant to SVDQuant", section "Smooth Quant (W8A8)") and weights
with a few magnified rows.  Every generator is seeded with
``numpy.random.PCG64(1000 + config_id)``; values are drawn in float64.
Activations are returned as float64 values that are already exactly
representable in bfloat16 (rounded to nearest-even here), because the layer
consumes bf16 activations.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_workload", "round_to_bf16", "small_case"]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    Input preparation only (the layer's activation dtype is bf16): uses the
    frexp/rint decomposition, exact in float64.  Values here are far from the
    bf16 overflow and subnormal ranges.
    """
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)                  # a = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


@dataclass
class Workload:
    """One seeded layer instance: X (M x K), W (K x N), bias (N), optional LoRA."""
    name: str
    M: int
    K: int
    N: int
    r: int
    alpha: float
    X: np.ndarray                      # float64, bf16-exact, M x K
    W: np.ndarray                      # float64, K x N
    bias: np.ndarray                   # float64, bf16-exact, N
    lora_A: Optional[np.ndarray] = None   # K x r_lora
    lora_B: Optional[np.ndarray] = None   # r_lora x N
    meta: dict = field(default_factory=dict)

    @property
    def r_eff(self) -> int:
        return self.r + (0 if self.lora_A is None else self.lora_A.shape[1])


def _outlier_channels(rng, X, count, lo, hi=None):
    idx = rng.choice(X.shape[1], size=count, replace=False)
    f = np.full(count, float(lo)) if hi is None else rng.uniform(lo, hi, size=count)
    X[:, idx] *= f[None, :]
    return idx


def _outlier_rows(rng, W, count, lo, hi=None):
    idx = rng.choice(W.shape[0], size=count, replace=False)
    f = np.full(count, float(lo)) if hi is None else rng.uniform(lo, hi, size=count)
    W[idx, :] *= f[:, None]
    return idx


def _tiny_recipe(rng, M, K, N, w_std):
    """First config's recipe: N(0,1) X with 4 channels x40, W rows: 4 random x8."""
    X = rng.standard_normal((M, K))
    xi = _outlier_channels(rng, X, 4, 40.0)
    W = rng.standard_normal((K, N)) * w_std
    wi = _outlier_rows(rng, W, 4, 8.0)
    return X, W, {"x_outlier_channels": xi.tolist(), "w_outlier_rows": wi.tolist()}


def make_workload(name: str, M: Optional[int] = None, seed_offset: int = 0) -> Workload:
    """Build a named workload.  ``M`` may be overridden (a row sample of the same layer).

    Names and recipes:
      tiny        M=256  K=512   N=512   r=32  X N(0,1), 4 channels x40; W N(0,1), 4 rows x8
      qkv         M=4608 K=3072  N=9216  r=32  X N(0,1), 1% channels x U(20,60); W N(0,0.02), 1% rows x U(20,60)
      fc1         M=4608 K=3072  N=12288 r=32  first-config recipe, W at N(0,0.02)
      fc2         M=4608 K=12288 N=3072  r=32  weights only (X is GELU of fc1's output, built by the caller)
      sweep_r{16,32,64}[_lora]  M=4096 K=N=4096, first-config recipe; LoRA rank 16, A,B ~ N(0,0.01)
      large       M=18432 K=3072 N=3072  r=32  X Student-t(3), 1% channels x50; W N(0,0.02)
    """
    ids = {"tiny": 1, "qkv": 2, "fc1": 3, "fc2": 3, "large": 5}
    if name.startswith("sweep"):
        cid = 4
    else:
        cid = ids[name]
    rng = np.random.Generator(np.random.PCG64(1000 + cid + seed_offset))
    lora_A = lora_B = None
    meta = {"config_id": cid}
    if name == "tiny":
        M0, K, N, r = 256, 512, 512, 32
        M = M or M0
        X, W, m = _tiny_recipe(rng, M, K, N, 1.0)
        meta.update(m)
        bias = rng.normal(0.0, 0.1, N)
    elif name == "qkv":
        M0, K, N, r = 4608, 3072, 9216, 32
        M = M or M0
        X = rng.standard_normal((M, K))
        meta["x_outlier_channels"] = _outlier_channels(rng, X, K // 100, 20.0, 60.0).tolist()
        W = rng.standard_normal((K, N)) * 0.02
        meta["w_outlier_rows"] = _outlier_rows(rng, W, K // 100, 20.0, 60.0).tolist()
        bias = rng.normal(0.0, 0.1, N)
    elif name in ("fc1", "fc2"):
        # one generator for the pair: fc1's draws first, then fc2's weight
        M = M or 4608
        X1, W1, m1 = _tiny_recipe(rng, M, 3072, 12288, 0.02)
        b1 = rng.normal(0.0, 0.1, 12288)
        W2 = rng.standard_normal((12288, 3072)) * 0.02
        w2i = _outlier_rows(rng, W2, 4, 8.0)
        b2 = rng.normal(0.0, 0.1, 3072)
        r = 32
        if name == "fc1":
            K, N, X, W, bias = 3072, 12288, X1, W1, b1
            meta.update(m1)
        else:
            K, N, W, bias = 12288, 3072, W2, b2
            X = np.zeros((M, K))        # placeholder: fc2's input is GELU(Y_fc1)
            meta["w_outlier_rows"] = w2i.tolist()
    elif name.startswith("sweep"):
        parts = name.split("_")
        r = int(parts[1][1:])
        M = M or 4096
        K = N = 4096
        X, W, m = _tiny_recipe(rng, M, K, N, 1.0)
        meta.update(m)
        bias = rng.normal(0.0, 0.1, N)
        if len(parts) > 2 and parts[2] == "lora":
            lora_A = rng.normal(0.0, 0.01, (K, 16))
            lora_B = rng.normal(0.0, 0.01, (16, N))
    elif name == "large":
        M0, K, N, r = 18432, 3072, 3072, 32
        M = M or M0
        X = rng.standard_t(3.0, (M, K))
        meta["x_outlier_channels"] = _outlier_channels(rng, X, K // 100, 50.0).tolist()
        W = rng.standard_normal((K, N)) * 0.02
        bias = rng.normal(0.0, 0.1, N)
    else:
        raise KeyError(name)
    return Workload(name=name, M=M, K=K, N=N, r=r, alpha=0.5,
                    X=round_to_bf16(X), W=W, bias=round_to_bf16(bias),
                    lora_A=lora_A, lora_B=lora_B, meta=meta)


def small_case(M: int, K: int, N: int, r: int, seed: int = 7, x_outliers: int = 2,
               w_outliers: int = 2) -> Workload:
    """A small seeded layer of arbitrary shape (tile, tail and edge-case tests)."""
    rng = np.random.Generator(np.random.PCG64(50_000 + seed))
    X = rng.standard_normal((M, K))
    if x_outliers and K > x_outliers:
        _outlier_channels(rng, X, x_outliers, 40.0)
    W = rng.standard_normal((K, N)) * 0.05
    if w_outliers and K > w_outliers:
        _outlier_rows(rng, W, w_outliers, 8.0)
    bias = rng.normal(0.0, 0.1, N)
    return Workload(name=f"small_{M}x{K}x{N}_r{r}", M=M, K=K, N=N, r=r, alpha=0.5,
                    X=round_to_bf16(X), W=W, bias=round_to_bf16(bias), meta={"seed": seed})


WORKLOADS = ("tiny", "qkv", "fc1", "fc2", "sweep_r16", "sweep_r32", "sweep_r64",
             "sweep_r16_lora", "sweep_r32_lora", "sweep_r64_lora", "large")
