"""Host-side checks of the packed layer (no GPU): tensors on the wrong device are refused before any
call reaches the library, which would otherwise be handed pointers the launching device cannot use."""
import pytest
import torch

from w4a4_rank_absorbed_b200.layer import check_device


def test_tensor_on_another_device_is_refused():
    with pytest.raises(ValueError, match="cpu"):
        check_device(torch.zeros(4), torch.device("cuda", 0), "X")
    with pytest.raises(ValueError):
        check_device(torch.zeros(4), torch.device("cuda", 1), "out")


def test_matching_device_and_missing_tensor_pass():
    check_device(None, torch.device("cuda", 0), "LAs")
    check_device(torch.zeros(4), torch.device("cpu"), "X")


def test_product_package_does_not_import_the_oracle():
    """The product path never reaches the oracle: importing the package and its modules pulls in no
    module of oracle/, and no product source names it in an import."""
    import pathlib
    import subprocess
    import sys
    root = pathlib.Path(__file__).resolve().parents[1]
    code = ("import sys; import w4a4_rank_absorbed_b200.layer, w4a4_rank_absorbed_b200.calib, "
            "w4a4_rank_absorbed_b200.svdq, w4a4_rank_absorbed_b200.synth; "
            "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]; "
            "assert not bad, bad")
    res = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    for f in (root / "w4a4_rank_absorbed_b200").rglob("*.py"):
        text = f.read_text()
        assert "import oracle" not in text and "from oracle" not in text, f


def test_no_copy_with_cluster_multicast_in_the_kernels():
    """No TMA or bulk copy in the library uses cluster multicast (the kernels stay legal for multi-GPU
    replicas, whose memory a multicast load could reach)."""
    import pathlib
    import re
    csrc = pathlib.Path(__file__).resolve().parents[1] / "w4a4_rank_absorbed_b200" / "csrc"
    for f in list(csrc.glob("*.cu")) + list(csrc.glob("*.cuh")):
        for line in f.read_text().splitlines():
            if re.search(r"cp\.async\.bulk", line):
                assert "multicast" not in line, (f.name, line)
