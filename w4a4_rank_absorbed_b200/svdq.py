"""Python binding of the C ABI in include/svdq.h (argument marshalling only).

Each function has the name of the C entry point it calls and forwards torch
CUDA tensors as raw device pointers; every step of the layer runs in the
CUDA library ``libsvdq.so`` built in-tree by ``w4a4_rank_absorbed_b200.build``.
There is no fallback: if the library is missing or the device is not an
sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libsvdq.so")
CHECK_LIB_PATH = os.path.join(_PKG_DIR, "libsvdq_check.so")   # debug build: every copy checked


def default_library_path() -> str:
    """libsvdq.so, or the library named by the SVDQ_LIBRARY environment variable ("check" selects the
    debug build libsvdq_check.so)."""
    v = os.environ.get("SVDQ_LIBRARY", "")
    if not v:
        return LIB_PATH
    return CHECK_LIB_PATH if v == "check" else v

SVDQ_OK = 0
SVDQ_ERR_INVALID_ARG = 1
SVDQ_ERR_UNSUPPORTED_SHAPE = 2
SVDQ_ERR_MISALIGNED = 3
SVDQ_ERR_CUDA = 4
SVDQ_ERR_TIMEOUT = 5
SVDQ_ERR_DEVICE = 6
SVDQ_ERR_SCRATCH = 7
SVDQ_ERR_CHECK = 8

EXPORTED = ("svdq_status_string", "svdq_version", "svdq_sf_bytes", "svdq_pack_weight", "svdq_quantize_act",
            "svdq_linear", "svdq_lowrank_down", "svdq_lowrank_up", "svdq_get_device_error", "svdq_linear_debug",
            "svdq_quantize_act_workspace_bytes", "svdq_dequant_weight", "svdq_quantize_act_noalloc",
            "svdq_mx_sf_bytes", "svdq_pack_weight_mx", "svdq_quantize_act_mx", "svdq_linear_mx",
            "svdq_linear_gelu_quantize", "svdq_linear_gelu_quantize_workspace_bytes", "svdq_gelu_bf16",
            "svdq_calib_absmax_cols", "svdq_calib_absmax_rows", "svdq_calib_smooth", "svdq_calib_scale_rows",
            "svdq_calib_act_amax", "svdq_map_cache_stats", "svdq_build_flags")


class SVDQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_lib: Optional[ctypes.CDLL] = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_F = ctypes.c_float


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libsvdq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or default_library_path()
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} (run python -m w4a4_rank_absorbed_b200.build)")
    lib = ctypes.CDLL(path)
    lib.svdq_status_string.restype = ctypes.c_char_p
    lib.svdq_status_string.argtypes = [_I]
    lib.svdq_version.restype = _I
    lib.svdq_version.argtypes = []
    lib.svdq_sf_bytes.restype = ctypes.c_size_t
    lib.svdq_sf_bytes.argtypes = [_I64, _I64]
    lib.svdq_pack_weight.restype = _I
    lib.svdq_pack_weight.argtypes = [_P, _P, _I64, _I64, _I, _P, _P, _P, ctypes.POINTER(_F), _P, _P]
    lib.svdq_quantize_act.restype = _I
    lib.svdq_quantize_act.argtypes = [_P, _I64, _I64, _P, _F, _P, _I, _F, _P, _P, _P, _P, ctypes.c_size_t, _P]
    lib.svdq_quantize_act_noalloc.restype = _I
    lib.svdq_quantize_act_noalloc.argtypes = [_P, _I64, _I64, _P, _F, _P, _I, _F, _P, _P, _P, _P]
    lib.svdq_quantize_act_workspace_bytes.restype = ctypes.c_size_t
    lib.svdq_quantize_act_workspace_bytes.argtypes = [_I64, _I64, _I]
    lib.svdq_linear.restype = _I
    lib.svdq_linear.argtypes = [_P, _P, _F, _P, _P, _F, _P, _P, _I, _P, _P, _I, _I64, _I64, _I64, _P]
    lib.svdq_linear_debug.restype = _I
    lib.svdq_linear_debug.argtypes = [_P, _P, _F, _P, _P, _F, _P, _P, _I, _P, _P, _I, _I64, _I64, _I64, _I,
                                      ctypes.c_uint64, _P]
    lib.svdq_dequant_weight.restype = _I
    lib.svdq_dequant_weight.argtypes = [_P, _P, _P, _I64, _I64, _P, _P]
    lib.svdq_lowrank_down.restype = _I
    lib.svdq_lowrank_down.argtypes = [_P, _I64, _I64, _P, _I, _F, _P, _P, ctypes.c_size_t, _P]
    lib.svdq_lowrank_up.restype = _I
    lib.svdq_lowrank_up.argtypes = [_P, _P, _I, _F, _P, _I, _I64, _I64, _P]
    lib.svdq_mx_sf_bytes.restype = ctypes.c_size_t
    lib.svdq_mx_sf_bytes.argtypes = [_I64, _I64]
    lib.svdq_pack_weight_mx.restype = _I
    lib.svdq_pack_weight_mx.argtypes = [_P, _P, _I64, _I64, _I, _P, _P, _P, _P]
    lib.svdq_quantize_act_mx.restype = _I
    lib.svdq_quantize_act_mx.argtypes = [_P, _I64, _I64, _P, _P, _I, _F, _P, _P, _P, _P, ctypes.c_size_t, _P]
    lib.svdq_linear_mx.restype = _I
    lib.svdq_linear_mx.argtypes = [_P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I64, _I64, _I64, _P]
    lib.svdq_linear_gelu_quantize_workspace_bytes.restype = ctypes.c_size_t
    lib.svdq_linear_gelu_quantize_workspace_bytes.argtypes = [_I64, _I64, _I]
    lib.svdq_linear_gelu_quantize.restype = _I
    lib.svdq_linear_gelu_quantize.argtypes = [_P, _P, _F, _P, _P, _F, _P, _P, _I, _P, _I64, _I64, _I64, _P, _F, _P, _I,
                                              _F, _P, _P, _P, _P, ctypes.c_size_t, _P]
    lib.svdq_gelu_bf16.restype = _I
    lib.svdq_gelu_bf16.argtypes = [_P, _I64, _P, _P]
    _D = ctypes.c_double
    for name, args in (("svdq_calib_absmax_cols", [_P, _I64, _I64, _P, _I, _P]),
                       ("svdq_calib_absmax_rows", [_P, _I64, _I64, _P, _P]),
                       ("svdq_calib_smooth", [_P, _P, _I64, _D, _P, _P, _P]),
                       ("svdq_calib_scale_rows", [_P, _P, _I64, _I64, _P, _P]),
                       ("svdq_calib_act_amax", [_P, _I64, _I64, _P, _P, _I, _P])):
        getattr(lib, name).restype = _I
        getattr(lib, name).argtypes = args
    lib.svdq_build_flags.restype = _I
    lib.svdq_build_flags.argtypes = []
    lib.svdq_map_cache_stats.restype = None
    lib.svdq_map_cache_stats.argtypes = [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64)]
    lib.svdq_get_device_error.restype = _I
    lib.svdq_get_device_error.argtypes = [_P, ctypes.POINTER(_I)]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load_library().svdq_status_string(int(status)).decode()
    except ImportError:
        return f"status {status}"


def _ptr(t: Optional[torch.Tensor], dtype=None, name: str = "") -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    return t.data_ptr()


def stream_handle(stream) -> int:
    """The cudaStream_t handle (as an int) of a torch stream or a raw handle."""
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != SVDQ_OK:
        raise SVDQError(status, where)


def svdq_sf_bytes(rows: int, K: int) -> int:
    return int(load_library().svdq_sf_bytes(rows, K))


def svdq_mx_sf_bytes(rows: int, K: int) -> int:
    return int(load_library().svdq_mx_sf_bytes(rows, K))


def svdq_pack_weight_mx(R, L2b, K, N, r, Wq, SFw, L2p, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_pack_weight_mx(_ptr(R, torch.float32, "R"), _ptr(L2b, torch.bfloat16, "L2b"), K, N, r,
                                 _ptr(Wq, torch.uint8, "Wq"), _ptr(SFw, torch.uint8, "SFw"),
                                 _ptr(L2p, torch.bfloat16, "L2p"), _stream(stream))
    _check(st, "svdq_pack_weight_mx")


def svdq_quantize_act_mx(X, M, K, inv_s, L1fT, r, lr_scale, Xq, SFx, LAs, workspace=None, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_quantize_act_mx(_ptr(X, torch.bfloat16, "X"), M, K, _ptr(inv_s, torch.float32, "inv_s"),
                                  _ptr(L1fT, torch.bfloat16, "L1fT"), r, float(lr_scale),
                                  _ptr(Xq, torch.uint8, "Xq"), _ptr(SFx, torch.uint8, "SFx"),
                                  _ptr(LAs, torch.bfloat16, "LAs"), _ptr(workspace, torch.uint8, "workspace"),
                                  _nbytes(workspace), _stream(stream))
    _check(st, "svdq_quantize_act_mx")


def svdq_linear_mx(Xq, SFx, Wq, SFw, LAs, L2p, r, bias, Y, y_fp32, M, N, K, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_linear_mx(_ptr(Xq, torch.uint8, "Xq"), _ptr(SFx, torch.uint8, "SFx"),
                            _ptr(Wq, torch.uint8, "Wq"), _ptr(SFw, torch.uint8, "SFw"),
                            _ptr(LAs, torch.bfloat16, "LAs"), _ptr(L2p, torch.bfloat16, "L2p"), r,
                            _ptr(bias, torch.bfloat16, "bias"), _ptr(Y, (torch.bfloat16, torch.float32), "Y"),
                            int(y_fp32), M, N, K, _stream(stream))
    _check(st, "svdq_linear_mx")


def svdq_linear_gelu_quantize_workspace_bytes(M: int, N: int, r2: int) -> int:
    return int(load_library().svdq_linear_gelu_quantize_workspace_bytes(M, N, r2))


def new_gelu_quantize_workspace(M: int, N: int, r2: int, device=None) -> Optional[torch.Tensor]:
    """Scratch for svdq_linear_gelu_quantize (None when none is needed); its contents need no initial value."""
    n = svdq_linear_gelu_quantize_workspace_bytes(M, N, r2)
    return torch.empty(n, dtype=torch.uint8, device=device if device is not None else "cuda") if n else None


def svdq_linear_gelu_quantize(Xq, SFx, gs_x, Wq, SFw, gs_w, LAs, L2p, r, bias, M, N, K, inv_s2, gs_x2, L1fT2, r2,
                              lr_scale2, Xq2, SFx2, LAs2, workspace=None, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_linear_gelu_quantize(
        _ptr(Xq, torch.uint8, "Xq"), _ptr(SFx, torch.uint8, "SFx"), float(gs_x), _ptr(Wq, torch.uint8, "Wq"),
        _ptr(SFw, torch.uint8, "SFw"), float(gs_w), _ptr(LAs, torch.bfloat16, "LAs"), _ptr(L2p, torch.bfloat16, "L2p"),
        r, _ptr(bias, torch.bfloat16, "bias"), M, N, K, _ptr(inv_s2, torch.float32, "inv_s2"), float(gs_x2),
        _ptr(L1fT2, torch.bfloat16, "L1fT2"), r2, float(lr_scale2), _ptr(Xq2, torch.uint8, "Xq2"),
        _ptr(SFx2, torch.uint8, "SFx2"), _ptr(LAs2, torch.bfloat16, "LAs2"), _ptr(workspace, torch.uint8, "workspace"),
        _nbytes(workspace), _stream(stream))
    _check(st, "svdq_linear_gelu_quantize")


def svdq_gelu_bf16(X, n, Y, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_gelu_bf16(_ptr(X, torch.bfloat16, "X"), n, _ptr(Y, torch.bfloat16, "Y"), _stream(stream))
    _check(st, "svdq_gelu_bf16")


def svdq_calib_absmax_cols(X, M, K, amax_x, accumulate=False, stream=None) -> None:
    _check(load_library().svdq_calib_absmax_cols(_ptr(X, torch.bfloat16, "X"), M, K, _ptr(amax_x, torch.float32, "amax_x"),
                                                 int(bool(accumulate)), _stream(stream)), "svdq_calib_absmax_cols")


def svdq_calib_absmax_rows(W, K, N, amax_w, stream=None) -> None:
    _check(load_library().svdq_calib_absmax_rows(_ptr(W, torch.float64, "W"), K, N, _ptr(amax_w, torch.float64, "amax_w"),
                                                 _stream(stream)), "svdq_calib_absmax_rows")


def svdq_calib_smooth(amax_x, amax_w, K, alpha, s, inv_s, stream=None) -> None:
    _check(load_library().svdq_calib_smooth(_ptr(amax_x, torch.float32, "amax_x"), _ptr(amax_w, torch.float64, "amax_w"),
                                            K, float(alpha), _ptr(s, torch.float64, "s"),
                                            _ptr(inv_s, torch.float32, "inv_s"), _stream(stream)), "svdq_calib_smooth")


def svdq_calib_scale_rows(W, s, K, N, W_hat, stream=None) -> None:
    _check(load_library().svdq_calib_scale_rows(_ptr(W, torch.float64, "W"), _ptr(s, torch.float64, "s"), K, N,
                                                _ptr(W_hat, torch.float64, "W_hat"), _stream(stream)),
           "svdq_calib_scale_rows")


def svdq_calib_act_amax(X, M, K, inv_s, amax, accumulate=False, stream=None) -> None:
    _check(load_library().svdq_calib_act_amax(_ptr(X, torch.bfloat16, "X"), M, K, _ptr(inv_s, torch.float32, "inv_s"),
                                              _ptr(amax, torch.float32, "amax"), int(bool(accumulate)),
                                              _stream(stream)), "svdq_calib_act_amax")


def svdq_map_cache_stats():
    """(hits, misses) of the library's tensor-map cache."""
    h, m = ctypes.c_uint64(0), ctypes.c_uint64(0)
    load_library().svdq_map_cache_stats(ctypes.byref(h), ctypes.byref(m))
    return int(h.value), int(m.value)


def svdq_build_flags() -> int:
    return int(load_library().svdq_build_flags())


def svdq_version() -> int:
    return int(load_library().svdq_version())


def svdq_pack_weight(R, L2b, K, N, r, Wq, SFw, gs_w, L2p, stream=None, sync: bool = True) -> Optional[float]:
    """Packs the residual weight.  With sync=True (the default) the call synchronises the stream and
    returns gs_w as a Python float (the library writes it to host memory); with sync=False it stays
    asynchronous and returns None (gs_w is then only in the device tensor)."""
    lib = load_library()
    host = _F(0.0)
    st = lib.svdq_pack_weight(_ptr(R, torch.float32, "R"), _ptr(L2b, torch.bfloat16, "L2b"), K, N, r,
                              _ptr(Wq, torch.uint8, "Wq"), _ptr(SFw, torch.uint8, "SFw"),
                              _ptr(gs_w, torch.float32, "gs_w"), ctypes.byref(host) if sync else None,
                              _ptr(L2p, torch.bfloat16, "L2p"), _stream(stream))
    _check(st, "svdq_pack_weight")
    return float(host.value) if sync else None


def svdq_quantize_act_noalloc(X, M, K, inv_s, gs_x, L1fT, r, lr_scale, Xq, SFx, LAs, stream=None) -> None:
    """svdq_quantize_act without a workspace: the library's own device scratch holds the partial sums
    (for callers that cannot allocate device memory; see include/svdq.h for the size limit)."""
    lib = load_library()
    st = lib.svdq_quantize_act_noalloc(_ptr(X, torch.bfloat16, "X"), M, K, _ptr(inv_s, torch.float32, "inv_s"),
                                       float(gs_x), _ptr(L1fT, torch.bfloat16, "L1fT"), r, float(lr_scale),
                                       _ptr(Xq, torch.uint8, "Xq"), _ptr(SFx, torch.uint8, "SFx"),
                                       _ptr(LAs, torch.bfloat16, "LAs"), _stream(stream))
    _check(st, "svdq_quantize_act_noalloc")


def svdq_quantize_act_workspace_bytes(M: int, K: int, r: int) -> int:
    return int(load_library().svdq_quantize_act_workspace_bytes(M, K, r))


def new_workspace(M: int, K: int, r: int, device=None) -> Optional[torch.Tensor]:
    """A zero-filled workspace for svdq_quantize_act / svdq_lowrank_down (None when none is needed)."""
    n = svdq_quantize_act_workspace_bytes(M, K, r)
    return torch.zeros(n, dtype=torch.uint8, device=device if device is not None else "cuda") if n else None


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def svdq_quantize_act(X, M, K, inv_s, gs_x, L1fT, r, lr_scale, Xq, SFx, LAs, workspace=None, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_quantize_act(_ptr(X, torch.bfloat16, "X"), M, K, _ptr(inv_s, torch.float32, "inv_s"),
                               float(gs_x), _ptr(L1fT, torch.bfloat16, "L1fT"), r, float(lr_scale),
                               _ptr(Xq, torch.uint8, "Xq"), _ptr(SFx, torch.uint8, "SFx"),
                               _ptr(LAs, torch.bfloat16, "LAs"), _ptr(workspace, torch.uint8, "workspace"),
                               _nbytes(workspace), _stream(stream))
    _check(st, "svdq_quantize_act")


def svdq_linear(Xq, SFx, gs_x, Wq, SFw, gs_w, LAs, L2p, r, bias, Y, y_fp32, M, N, K, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_linear(_ptr(Xq, torch.uint8, "Xq"), _ptr(SFx, torch.uint8, "SFx"), float(gs_x),
                         _ptr(Wq, torch.uint8, "Wq"), _ptr(SFw, torch.uint8, "SFw"), float(gs_w),
                         _ptr(LAs, torch.bfloat16, "LAs"), _ptr(L2p, torch.bfloat16, "L2p"), r,
                         _ptr(bias, torch.bfloat16, "bias"), _ptr(Y, (torch.bfloat16, torch.float32), "Y"),
                         int(y_fp32), M, N, K, _stream(stream))
    _check(st, "svdq_linear")


def svdq_linear_debug(Xq, SFx, gs_x, Wq, SFw, gs_w, LAs, L2p, r, bias, Y, y_fp32, M, N, K, debug_flags,
                      timeout_ns, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_linear_debug(_ptr(Xq, torch.uint8, "Xq"), _ptr(SFx, torch.uint8, "SFx"), float(gs_x),
                               _ptr(Wq, torch.uint8, "Wq"), _ptr(SFw, torch.uint8, "SFw"), float(gs_w),
                               _ptr(LAs, torch.bfloat16, "LAs"), _ptr(L2p, torch.bfloat16, "L2p"), r,
                               _ptr(bias, torch.bfloat16, "bias"), _ptr(Y, (torch.bfloat16, torch.float32), "Y"),
                               int(y_fp32), M, N, K, int(debug_flags), int(timeout_ns), _stream(stream))
    _check(st, "svdq_linear_debug")


def svdq_dequant_weight(Wq, SFw, gs_w, K, N, Rq, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_dequant_weight(_ptr(Wq, torch.uint8, "Wq"), _ptr(SFw, torch.uint8, "SFw"),
                                 _ptr(gs_w, torch.float32, "gs_w"), K, N, _ptr(Rq, torch.float32, "Rq"),
                                 _stream(stream))
    _check(st, "svdq_dequant_weight")


def svdq_lowrank_down(X, M, K, L1fT, r, lr_scale, LAs, workspace, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_lowrank_down(_ptr(X, torch.bfloat16, "X"), M, K, _ptr(L1fT, torch.bfloat16, "L1fT"), r,
                               float(lr_scale), _ptr(LAs, torch.bfloat16, "LAs"),
                               _ptr(workspace, torch.uint8, "workspace"), _nbytes(workspace), _stream(stream))
    _check(st, "svdq_lowrank_down")


def svdq_lowrank_up(LAs, L2p, r, gs, Y, y_fp32, M, N, stream=None) -> None:
    lib = load_library()
    st = lib.svdq_lowrank_up(_ptr(LAs, torch.bfloat16, "LAs"), _ptr(L2p, torch.bfloat16, "L2p"), r, float(gs),
                             _ptr(Y, (torch.bfloat16, torch.float32), "Y"), int(y_fp32), M, N, _stream(stream))
    _check(st, "svdq_lowrank_up")


def svdq_get_device_error(stream=None):
    """Returns (status, site); clears the device error word."""
    lib = load_library()
    site = _I(0)
    st = lib.svdq_get_device_error(_stream(stream), ctypes.byref(site))
    return int(st), int(site.value)
