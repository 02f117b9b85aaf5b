"""CPU oracle for the SVDQuant W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct statement of what the
layer computes, written from the method's description and used to check the
CUDA path.  It is not part of the product: only the test suite, the smoke
check of ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may
import it.  It shares no code with the CUDA library and imports nothing
from the product package.

Arithmetic: float64 for the matrix products and the decomposition; the
quantizer's decisions (which E2M1 code, which UE4M3 scale) are taken in
IEEE binary32, the precision the GPU kernels decide them in, using numpy
float32 operations (each correctly rounded).

Sources (page title, section):
  * "SVDQuant" review (jeonghoonpark.com): §3 Quantization Preliminary
    (absmax quantizer, q_max = 6 for 4-bit FP, scaled product),
    §4.1 Problem Formulation (the four error factors), §4.2 (smoothing,
    low-rank branch L1 = U Sigma_r, L2 = V_r^T, residual R, the output
    decomposition), §4.3 Nunchaku (kernel fusion).
  * "From SmoothQuant to SVDQuant" (ch3chohch3.github.io): section Smooth
    Quant (W8A8) (smoothing equation and the per-channel factor with alpha),
    section SVDQuant (W4A4) / SVD decomposition and quantization scheme
    (rank 32 default, L1/L2 shapes, static weight-side quantities),
    section Personal view (NVFP4: group 16 with a two-level scale).
  * "SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit
    Diffusion Models" (abstract): LoRA added to the low-rank branch without
    re-quantization.

Parity status of each function is given in its module's header.
"""
