"""Shared helpers of the parity tests: per-slice relative L2 error and tensor conversion."""
import numpy as np


def f64(t):
    """A torch tensor (any device/dtype) or array as float64 numpy."""
    if hasattr(t, "detach"):
        return t.detach().double().cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def max_rel_l2(x, ref, lead: int):
    """max over the leading `lead` axes of ||x - ref||_2 / ||ref||_2 (the per-(b,h)-slice
    relative L2 error); a zero reference slice compares absolute error instead."""
    x, ref = f64(x), f64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    xs = x.reshape(int(np.prod(x.shape[:lead])) if lead else 1, -1)
    rs = ref.reshape(xs.shape)
    num = np.linalg.norm(xs - rs, axis=1)
    den = np.linalg.norm(rs, axis=1)
    return float(np.max(np.where(den > 0, num / np.where(den > 0, den, 1), num)))


CANARY = 0xA5
GUARD_BYTES = 4096


def guarded(shape, dtype, device):
    """A contiguous tensor of `shape` inside a larger buffer whose GUARD_BYTES before and after
    hold the byte CANARY (a stand-in for a memory sanitizer: a kernel writing past its output
    changes a guard byte). The view starts GUARD_BYTES into the buffer, so it keeps the buffer's
    alignment. Returns (view, buffer)."""
    import torch

    elem = torch.empty((), dtype=dtype).element_size()
    n = 1
    for s in shape:
        n *= s
    pad = GUARD_BYTES // elem
    buf = torch.empty(n + 2 * pad, dtype=dtype, device=device)
    buf.view(torch.uint8).fill_(CANARY)
    return buf[pad:pad + n].view(shape), buf


def guards_intact(view, buf) -> bool:
    """True if no byte outside `view` in `buf` has changed from CANARY."""
    import torch

    raw = buf.view(torch.uint8)
    start = (view.data_ptr() - buf.data_ptr())
    end = start + view.numel() * view.element_size()
    return bool((raw[:start] == CANARY).all()) and bool((raw[end:] == CANARY).all())
