"""The guarded-buffer helper itself, on the CPU: writes that fit leave the guards intact,
one element past either end does not, and the inner tensor is aligned and holds its data."""
import torch

from tests.canary import GUARD_BYTES, Guarded, guarded_like


def test_writes_inside_keep_the_guards():
    g = Guarded((3, 5, 8), torch.bfloat16, "cpu")
    g.tensor.fill_(1.5)
    assert g.intact()
    assert g.tensor.data_ptr() % 16 == 0 and g.tensor.is_contiguous()


def test_one_element_past_either_end_is_seen():
    for dtype in (torch.float32, torch.bfloat16, torch.int32):
        g = Guarded((4, 6), dtype, "cpu")
        assert g.intact()
        g.buf[GUARD_BYTES + g.nbytes] = 0   # first byte after the tensor
        assert not g.intact()
        g = Guarded((4, 6), dtype, "cpu")
        g.buf[GUARD_BYTES - 1] = 0          # last byte before it
        assert not g.intact()


def test_initial_data_is_copied_in():
    src = torch.randn(2, 7, 3)
    g = guarded_like(src)
    assert torch.equal(g.tensor, src) and g.intact()


def test_empty_tensor():
    g = Guarded((0, 4), torch.float32, "cpu")
    assert g.tensor.numel() == 0 and g.intact()
