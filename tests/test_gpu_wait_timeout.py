"""A pipeline wait that runs out is reported, and leaves the device usable.

Every wait of the dual-form kernels on an mbarrier phase is bounded; one that gives up sets bit 0
of the device error word, and the kernel's warps leave their loops together (copies and MMAs
already in flight are still waited for) instead of hanging. Here the limit of the stage kernel
is cut to 1 ns through the library's tuning choice, so that waits run out in an otherwise normal
call (no fault, trap or endless loop is involved); the next call with the normal limit must be
exact.
"""
import os

import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu


def run(x):
    return ttt.ttt_linear_dual_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"], C=16)


def test_timed_out_wait_sets_the_error_bit_and_the_next_call_is_exact(cuda_lib, tuning):
    # The limit is checked between hardware try-waits, which suspend the thread for a while on
    # their own before reporting an incomplete phase; 512 pipeline stages per stream give the
    # stage kernel's issue and epilogue warps hundreds of waits of a whole stage's chain time.
    x = inp.dual_or_assoc_inputs(1, 2, 65536, 64, seed=91, device="cuda", normalise=("K", "V"))
    assert ttt.read_device_error() == 0
    tuning("dual_kernel", 3)
    tuning("wait_limit_ns", 1)
    run(x)   # the launch itself succeeds; the give-up is reported on the device
    err = ttt.read_device_error()
    assert err & 1, err
    assert ttt.read_device_error() == 0   # the read cleared the word
    tuning("wait_limit_ns", 0)
    O, W = run(x)
    assert ttt.read_device_error() == 0
    Q, K, V = (x[k].float().cpu().numpy() for k in ("Q", "K", "V"))
    Or, Wr = orc.dual_form(Q, K, V, x["eta"].cpu().numpy(), x["W0"].cpu().numpy(), 16,
                           threads=os.cpu_count() or 4)
    assert max_rel_l2(O, Or, 2) <= 1e-2 and max_rel_l2(W, Wr, 2) <= 1e-2
