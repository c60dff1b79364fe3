"""The guard-band helper of the GPU canary tests, checked on the CPU: an untouched buffer passes,
a write one element past either end of the view is caught, and the view is aligned and
contiguous."""
import torch

from _helpers import GUARD_BYTES, guarded, guards_intact


def test_guard_bands_catch_writes_past_either_end():
    for dtype in (torch.float32, torch.bfloat16, torch.uint8):
        v, buf = guarded((3, 5, 8), dtype, "cpu")
        assert v.is_contiguous() and v.shape == (3, 5, 8)
        assert (v.data_ptr() - buf.data_ptr()) == GUARD_BYTES
        v.fill_(1)                       # writing the whole view is fine
        assert guards_intact(v, buf)
        flat = buf.view(-1)
        pad = GUARD_BYTES // v.element_size()
        flat[pad + v.numel()] = 2        # one element past the end
        assert not guards_intact(v, buf)
        v2, buf2 = guarded((4,), dtype, "cpu")
        buf2.view(-1)[GUARD_BYTES // v2.element_size() - 1] = 3   # one element before the start
        assert not guards_intact(v2, buf2)
