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
