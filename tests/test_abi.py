"""The C ABI library loads, exports every declared symbol and validates arguments (CPU only)."""
import os
import re

import pytest

from w4a4_rank_absorbed_b200 import build, svdq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return svdq.load_library()


def _declared():
    text = open(os.path.join(ROOT, "include", "svdq.h")).read()
    return sorted(set(re.findall(r"SVDQ_API\s+[\w\s\*]+?\b(svdq_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(svdq.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings_and_sizes(lib):
    assert svdq.status_string(0) == "SVDQ_OK"
    assert svdq.status_string(5) == "SVDQ_ERR_TIMEOUT"
    assert svdq.svdq_version() >= 100
    assert svdq.svdq_sf_bytes(256, 512) == 256 * 32
    assert svdq.svdq_sf_bytes(200, 512) == 256 * 32
    assert svdq.svdq_sf_bytes(1, 64) == 128 * 4
    assert svdq.svdq_sf_bytes(10, 100) == 0


def test_workspace_size_query(lib):
    # ticket words (one per 128-row block, padded to 256 bytes), then up to 8 partial sums of M x r floats
    assert svdq.svdq_quantize_act_workspace_bytes(4608, 3072, 0) == 0
    assert svdq.svdq_quantize_act_workspace_bytes(4608, 3072, 32) == 256 + 8 * 4608 * 32 * 4
    assert svdq.svdq_quantize_act_workspace_bytes(200, 512, 16) == 256 + 8 * 256 * 16 * 4
    assert svdq.svdq_quantize_act_workspace_bytes(100, 96, 16) == 0        # K % 64: rejected shape
    assert svdq.svdq_quantize_act_workspace_bytes(100, 128, 24) == 0       # r % 16


def _linear(lib, **kw):
    a = dict(Xq=16, SFx=16, gs_x=1.0, Wq=16, SFw=16, gs_w=1.0, LAs=16, L2p=16, r=32, bias=None, Y=16,
             y_fp32=0, M=128, N=256, K=256, stream=None)
    a.update(kw)
    return lib.svdq_linear(a["Xq"], a["SFx"], a["gs_x"], a["Wq"], a["SFw"], a["gs_w"], a["LAs"], a["L2p"],
                           a["r"], a["bias"], a["Y"], a["y_fp32"], a["M"], a["N"], a["K"], a["stream"])


def test_argument_errors_before_any_launch(lib):
    assert _linear(lib, K=96) == svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _linear(lib, N=24) == svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _linear(lib, r=8) == svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _linear(lib, r=144) == svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _linear(lib, M=-1) == svdq.SVDQ_ERR_INVALID_ARG
    assert _linear(lib, M=0) == svdq.SVDQ_OK                 # an empty batch launches nothing
    assert _linear(lib, M=1 << 31) == svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _linear(lib, Xq=None) == svdq.SVDQ_ERR_INVALID_ARG
    assert _linear(lib, LAs=None) == svdq.SVDQ_ERR_INVALID_ARG
    assert _linear(lib, LAs=None, L2p=None, r=0) != svdq.SVDQ_ERR_INVALID_ARG
    assert _linear(lib, y_fp32=2) == svdq.SVDQ_ERR_INVALID_ARG
    assert _linear(lib, Y=24) == svdq.SVDQ_ERR_MISALIGNED
    assert _linear(lib, bias=8) == svdq.SVDQ_ERR_MISALIGNED
    ws = svdq.svdq_quantize_act_workspace_bytes(64, 128, 32)
    assert lib.svdq_quantize_act(16, 64, 100, 16, 1.0, 16, 32, 1.0, 16, 16, 16, 16, ws, None) == \
        svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert lib.svdq_quantize_act(16, 64, 128, 16, 1.0, None, 32, 1.0, 16, 16, 16, 16, ws, None) == \
        svdq.SVDQ_ERR_INVALID_ARG
    # a workspace missing or smaller than the query says
    assert lib.svdq_quantize_act(16, 64, 128, 16, 1.0, 16, 32, 1.0, 16, 16, 16, None, 0, None) == \
        svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_quantize_act(16, 64, 128, 16, 1.0, 16, 32, 1.0, 16, 16, 16, 16, ws - 1, None) == \
        svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_lowrank_down(16, 64, 128, 16, 0, 1.0, 16, 16, ws, None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_lowrank_down(16, 64, 128, 16, 32, 1.0, 16, 8, ws, None) == svdq.SVDQ_ERR_MISALIGNED
    assert lib.svdq_lowrank_up(16, 16, 0, 1.0, 16, 0, 64, 64, None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_lowrank_up(16, 16, 32, 1.0, 16, 0, 64, 40, None) == svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert lib.svdq_pack_weight(16, 16, 128, 40, 32, 16, 16, 16, None, 16, None) == svdq.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert lib.svdq_pack_weight(4, 16, 128, 32, 32, 16, 16, 16, None, 16, None) == svdq.SVDQ_ERR_MISALIGNED
    for flags in (2, 4, 8):        # only bit 0 is defined
        assert lib.svdq_linear_debug(16, 16, 1.0, 16, 16, 1.0, 16, 16, 32, None, 16, 0, 128, 256, 256, flags, 0,
                                     None) == svdq.SVDQ_ERR_INVALID_ARG


def test_valid_arguments_without_a_gpu_report_a_device_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _linear(lib) in (svdq.SVDQ_ERR_CUDA, svdq.SVDQ_ERR_DEVICE)


def test_empty_batch_is_a_no_op_and_shape_errors_still_apply():
    """M = 0 launches nothing (no CUDA call, so this runs without a GPU) and returns SVDQ_OK with NULL
    buffers; shape errors of the other dimensions are still reported."""
    from w4a4_rank_absorbed_b200 import svdq as C
    lib = C.load_library()
    OK, UNSUP, INVAL = C.SVDQ_OK, C.SVDQ_ERR_UNSUPPORTED_SHAPE, C.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_quantize_act(None, 0, 256, None, 1.0, None, 32, 1.0, None, None, None, None, 0, None) == OK
    assert lib.svdq_quantize_act(None, 0, 100, None, 1.0, None, 32, 1.0, None, None, None, None, 0, None) == UNSUP
    assert lib.svdq_quantize_act_noalloc(None, 0, 256, None, 1.0, None, 16, 1.0, None, None, None, None) == OK
    assert lib.svdq_linear(None, None, 1.0, None, None, 1.0, None, None, 32, None, None, 0, 0, 512, 256, None) == OK
    assert lib.svdq_linear(None, None, 1.0, None, None, 1.0, None, None, 32, None, None, 0, 0, 500, 256, None) == UNSUP
    assert lib.svdq_lowrank_down(None, 0, 256, None, 32, 1.0, None, None, 0, None) == OK
    assert lib.svdq_lowrank_down(None, 0, 256, None, 0, 1.0, None, None, 0, None) == INVAL
    assert lib.svdq_lowrank_up(None, None, 32, 1.0, None, 0, 0, 512, None) == OK
    assert lib.svdq_quantize_act_mx(None, 0, 256, None, None, 0, 1.0, None, None, None, None, 0, None) == OK
    assert lib.svdq_quantize_act_mx(None, 0, 192, None, None, 0, 1.0, None, None, None, None, 0, None) == UNSUP
    assert lib.svdq_linear_mx(None, None, None, None, None, None, 0, None, None, 0, 0, 256, 192, None) == UNSUP
    assert lib.svdq_linear_gelu_quantize(None, None, 1.0, None, None, 1.0, None, None, 0, None, 0, 512, 256, None,
                                         1.0, None, 32, 1.0, None, None, None, None, 0, None) == OK
    assert lib.svdq_linear_gelu_quantize(None, None, 1.0, None, None, 1.0, None, None, 0, None, 0, 512, 256, None,
                                         1.0, None, 48, 1.0, None, None, None, None, 0, None) == UNSUP
    assert lib.svdq_quantize_act(None, -1, 256, None, 1.0, None, 0, 1.0, None, None, None, None, 0, None) == INVAL


def test_plain_c_client_compiles_against_the_header_and_runs(tmp_path):
    """include/svdq.h compiles as strict C99 and a C program linked to libsvdq.so gets the documented
    answers from the calls that need no GPU (sizes, argument errors, empty batches)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    from w4a4_rank_absorbed_b200 import svdq
    svdq.load_library()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.dirname(svdq.LIB_PATH)
    exe = str(tmp_path / "svdq_client")
    build = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                            "-I", os.path.join(root, "include"), os.path.join(root, "tests", "c_client", "svdq_client.c"),
                            "-L", lib_dir, "-l:libsvdq.so", "-Wl,-rpath," + lib_dir, "-o", exe],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "c client ok" in run.stdout, run.stdout + run.stderr
