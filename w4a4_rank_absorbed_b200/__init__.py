"""B200-native (sm_100a) SVDQuant W4A4 linear layer.

    svdq      -- binding of the C ABI (include/svdq.h) of libsvdq.so
    layer     -- SVDQLinear: packed layer, forward = quantize_act + linear
    calib     -- offline smoothing / SVD / residual decomposition (float64, host)
    synth     -- seeded synthetic workloads
    build     -- nvcc build of libsvdq.so (in-tree)
"""
__all__ = ["svdq", "layer", "calib", "synth", "build"]
