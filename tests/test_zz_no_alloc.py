"""The entry point for callers that cannot allocate device memory (svdq_quantize_act_noalloc).

Such callers cannot hand the library a workspace: for example a host application whose memory pool
owns all of the GPU's memory, or a runtime that must not allocate once it runs.  The entry point keeps
the K-split's partial sums in a scratch array the library itself holds in device memory.  Its outputs
must equal those of svdq_quantize_act with a caller workspace, call after call (the array keeps the
previous call's contents, so a second call in a row checks that nothing stale leaks into the next one).

This file is collected last so that a run stopping at the first failure has run everything else.
"""
import numpy as np
import pytest
import torch

from helpers import bf16_dev, check_las, oracle_layer, require_gpu
from w4a4_rank_absorbed_b200.synth import small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _outputs(C, M, K, r):
    Xq = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    SFx = torch.empty(C.svdq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
    LAs = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda") if r else None
    return Xq, SFx, LAs


@pytest.mark.parametrize("M,K,r", [(1152, 3072, 32), (300, 1024, 64), (4608, 3072, 32), (37, 256, 16),
                                   (640, 512, 0)])
def test_noalloc_matches_the_workspace_entry_point(M, K, r):
    from w4a4_rank_absorbed_b200 import svdq as C
    wl = small_case(M, K, 128, r, seed=M + K + r)
    dec = oracle_layer(wl, r)
    assert dec.L1f.shape[1] == r
    X = bf16_dev(wl.X)
    inv_s = torch.from_numpy(dec.inv_s).cuda()
    L1fT = bf16_dev(np.ascontiguousarray(dec.L1f.T)) if r else None
    gs_x = float(np.float32(dec.gs_x))
    lr_scale = 1.0 / 64.0
    ref = _outputs(C, M, K, r)
    C.svdq_quantize_act(X, M, K, inv_s, gs_x, L1fT, r, lr_scale, *ref, C.new_workspace(M, K, r))
    for call in range(2):                   # two calls in a row share the library's scratch
        got = _outputs(C, M, K, r)
        C.svdq_quantize_act_noalloc(X, M, K, inv_s, gs_x, L1fT, r, lr_scale, *got)
        torch.cuda.synchronize()
        assert C.svdq_get_device_error()[0] == 0
        assert torch.equal(got[0], ref[0]), f"call {call}: codes"
        assert torch.equal(got[1], ref[1]), f"call {call}: scales"
        if r:
            assert torch.equal(got[2].view(torch.int16), ref[2].view(torch.int16)), f"call {call}: LAs"
            check_las(got[2], wl.X, dec.L1f, lr_scale)


def test_noalloc_refuses_a_shape_beyond_its_scratch():
    from w4a4_rank_absorbed_b200 import svdq as C
    # M = 4608 at r = 128 splits K over 4 CTAs a row block: 4 x 4608 x 128 x 4 bytes of partial sums,
    # more than the library's 8 MiB.  Refused before anything is launched.
    M, K, r = 4608, 3072, 128
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    inv_s = torch.ones(K, device="cuda")
    L1fT = torch.zeros((r, K), dtype=torch.bfloat16, device="cuda")
    out = _outputs(C, M, K, r)
    with pytest.raises(C.SVDQError) as e:
        C.svdq_quantize_act_noalloc(X, M, K, inv_s, 1.0, L1fT, r, 1.0, *out)
    assert e.value.status == C.SVDQ_ERR_SCRATCH
