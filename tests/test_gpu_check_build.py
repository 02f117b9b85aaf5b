"""The debug build (libsvdq_check.so): the small parity suites pass under it with no copy check firing,
and a planted misaligned box (a test hook only that build accepts) is caught by its check and reported
as SVDQ_ERR_CHECK instead of being issued."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from helpers import require_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    from w4a4_rank_absorbed_b200 import build
    build.build(check=True)


def _run(code: str, timeout=900):
    env = dict(os.environ, SVDQ_LIBRARY="check")
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_parity_suites_pass_under_the_check_build():
    env = dict(os.environ, SVDQ_LIBRARY="check")
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu and not slow",
                          "tests/test_gpu_parity.py", "tests/test_gpu_mx.py", "tests/test_gpu_mlp.py",
                          "-k", "not check_build"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-2000:]


def test_planted_misaligned_box_is_caught():
    code = r'''
import numpy as np, torch
from w4a4_rank_absorbed_b200 import svdq as C
assert C.svdq_build_flags() & 1, "not the check build"
M, N, K = 128, 256, 256
dev = torch.device("cuda", 0)
Xq = torch.zeros((M, K // 2), dtype=torch.uint8, device=dev)
Wq = torch.zeros((N, K // 2), dtype=torch.uint8, device=dev)
SFx = torch.zeros(C.svdq_sf_bytes(M, K), dtype=torch.uint8, device=dev)
SFw = torch.zeros(C.svdq_sf_bytes(N, K), dtype=torch.uint8, device=dev)
Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
C.svdq_linear_debug(Xq, SFx, 1.0, Wq, SFw, 1.0, None, None, 0, None, Y, 0, M, N, K, 2, 2_000_000)
st, site = C.svdq_get_device_error()
assert st == C.SVDQ_ERR_CHECK and site == 0x3c1, (st, hex(site))
# the context is still usable: a normal call afterwards is clean
C.svdq_linear(Xq, SFx, 1.0, Wq, SFw, 1.0, None, None, 0, None, Y, 0, M, N, K)
st, site = C.svdq_get_device_error()
assert st == 0, (st, hex(site))
print("caught")
'''
    res = _run(code)
    assert res.returncode == 0 and "caught" in res.stdout, res.stdout[-2000:] + res.stderr[-2000:]


def test_regular_build_refuses_the_planted_box():
    from w4a4_rank_absorbed_b200 import svdq as C
    if C.svdq_build_flags() & 1:
        pytest.skip("the check build is loaded in this process")
    d = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    Y = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(C.SVDQError) as e:
        C.svdq_linear_debug(d, d, 1.0, d, d, 1.0, None, None, 0, None, Y, 0, 128, 256, 256, 2, 2_000_000)
    assert e.value.status == C.SVDQ_ERR_INVALID_ARG
