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
