"""CPU: the canary helper detects what it is meant to detect (a write just
before or just after a buffer, an element left unwritten), so a green GPU
canary test means the calls really stayed inside their buffers."""
import torch

from canary import Guarded, GuardedWorkspace


def test_guard_bands_catch_writes_on_either_side():
    for dt in (torch.float32, torch.int32, torch.bfloat16):
        g = Guarded((3, 5), dt, "cpu")
        assert g.intact() and g.untouched() == 15
        g.t.zero_()
        assert g.intact() and g.untouched() == 0
        g._raw[g.guard - 1] ^= 1                       # last byte before the tensor
        assert not g.intact()
        h = Guarded((7,), dt, "cpu")
        h._raw[h.guard + h.nbytes] ^= 1                # first byte after it
        assert not h.intact()


def test_unwritten_elements_are_counted_and_nan_filled():
    g = Guarded((4, 4), torch.float32, "cpu")
    assert torch.isnan(g.t).all()
    g.t[:3] = 1.0
    assert g.untouched() == 4
    b = Guarded((8,), torch.bfloat16, "cpu")
    assert torch.isnan(b.t.float()).all()


def test_workspace_has_exactly_the_requested_size():
    w = GuardedWorkspace(1000, "cpu")
    assert w.t.numel() == 1000 and w.t.data_ptr() - w.buf.data_ptr() == w.guard
    w.t.fill_(0)
    assert w.intact()
    w._raw[w.guard + 1000] = 0
    assert not w.intact()
