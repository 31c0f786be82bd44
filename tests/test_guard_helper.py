"""The guard-band helper itself (CPU): writes inside the tensor leave the
margins intact; one element written just past either end is detected."""
import pytest
import torch

from guard import guarded


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.uint8])
def test_writes_inside_keep_the_margins(dtype):
    v, intact = guarded((3, 5, 7), dtype, "cpu", fill=torch.ones((3, 5, 7), dtype=dtype))
    assert v.is_contiguous() and v.shape == (3, 5, 7) and v.data_ptr() % 16 == 0
    assert bool((v == 1).all()) and intact()
    v.zero_()
    assert intact()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.uint8])
def test_one_element_past_either_end_is_detected(dtype):
    v, intact = guarded((4, 6), dtype, "cpu")
    past_end = torch.as_strided(v, (v.numel() + 1,), (1,), v.storage_offset())
    past_end[-1] = 0
    assert not intact()
    v, intact = guarded((4, 6), dtype, "cpu")
    before = torch.as_strided(v, (1,), (1,), v.storage_offset() - 1)
    before[0] = 0
    assert not intact()
