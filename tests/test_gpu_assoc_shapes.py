"""GPU parity of the associative mode at head dim 64 and chunk sizes 16 and 32, through the C ABI:
forward, backward, momentum and the state-only pass, against the fp64 oracle.

The associative recurrence is per token, so the chunk size does not change the result; the
oracle runs each case at the caller's C (its chunk form is pinned to the sequential recurrence
in tests/test_oracle_pins.py). Tolerance: per-(b,h) relative L2 <= 1e-2, as for d = 128, C = 64.
"""
import os

import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu
TOL = 1e-2
THREADS = os.cpu_count() or 4


def make(B, H, T, d, seed, eta="sigmoid"):
    x = inp.dual_or_assoc_inputs(B, H, T, d, seed=seed, device="cuda", normalise=("Q", "K"),
                                 eta=eta, eta_const=0.25, w0="zero")
    g = torch.Generator("cuda").manual_seed(seed + 1)
    x["S0"] = torch.randn(B, H, d, d, device="cuda", generator=g) * 0.05
    x["M0"] = torch.randn(B, H, d, d, device="cuda", generator=g) * 0.05
    x["dO"] = torch.randn(B, H, T, d, device="cuda", generator=g).to(torch.bfloat16)
    x["dS_out"] = torch.randn(B, H, d, d, device="cuda", generator=g) * 0.05
    return x


def np_(t):
    return None if t is None else t.float().cpu().numpy()


def eta_of(x):
    return x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("parts", [1, 4])
def test_forward(cuda_lib, tuning, d, C, parts):
    """One and four superchunks per stream (prefix scan over parts), a given S0."""
    tuning("assoc_parts", parts)
    x = make(2, 3, 1024, d, seed=d + C + parts)
    O, S = ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], x["eta"], x["S0"], C=C)
    Or, Sr = orc.assoc_scan(np_(x["Q"]), np_(x["K"]), np_(x["V"]), eta_of(x), np_(x["S0"]),
                            form="chunked", C=C, threads=THREADS)
    eo, es = max_rel_l2(O, Or, 2), max_rel_l2(S, Sr, 2)
    assert eo <= TOL and es <= TOL, (eo, es)
    assert ttt.read_device_error() == 0


def test_forward_d64_scalar_rate_zero_state_and_chunk_independence(cuda_lib):
    """The three chunk sizes give the same bits (they run on the same 64-token tiles)."""
    x = make(1, 4, 512, 64, seed=7, eta="const")
    outs = [ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], None, None, C=C,
                                   eta_scalar=x["eta_scalar"]) for C in (16, 32, 64)]
    for O, S in outs[1:]:
        assert torch.equal(O, outs[0][0]) and torch.equal(S, outs[0][1])
    Or, Sr = orc.assoc_scan(np_(x["Q"]), np_(x["K"]), np_(x["V"]), x["eta_scalar"], None,
                            threads=THREADS)
    assert max_rel_l2(outs[0][0], Or, 2) <= TOL and max_rel_l2(outs[0][1], Sr, 2) <= TOL


@pytest.mark.parametrize("d,C", [(64, 16), (64, 64), (128, 32)])
def test_backward(cuda_lib, d, C):
    x = make(1, 2, 640, d, seed=d * 3 + C)
    got = ttt.ttt_assoc_scan_bwd(x["Q"], x["K"], x["V"], x["eta"], x["S0"], x["dO"],
                                 x["dS_out"], C=C)
    ref = orc.assoc_scan_bwd(np_(x["Q"]), np_(x["K"]), np_(x["V"]), eta_of(x), np_(x["S0"]),
                             np_(x["dO"]), np_(x["dS_out"]), threads=THREADS)
    for name, g, r in zip(("dQ", "dK", "dV", "deta", "dS0"), got, ref):
        e = max_rel_l2(g, r, 2)
        assert e <= TOL, (name, e)
    assert ttt.read_device_error() == 0


@pytest.mark.parametrize("d,C", [(64, 32), (128, 16)])
def test_momentum(cuda_lib, d, C):
    x = make(1, 2, 512, d, seed=d + 5 * C)
    got = ttt.ttt_assoc_momentum_fwd(x["Q"], x["K"], x["V"], x["eta"], 0.5, x["S0"], x["M0"],
                                     C=C)
    ref = orc.assoc_momentum(np_(x["Q"]), np_(x["K"]), np_(x["V"]), eta_of(x), 0.5,
                             np_(x["S0"]), np_(x["M0"]), threads=THREADS)
    for name, g, r in zip(("O", "S", "M"), got, ref):
        e = max_rel_l2(g, r, 2)
        assert e <= TOL, (name, e)


def test_state_pass_d64(cuda_lib):
    """The context-parallel state increment sum_t eta_t k_t^T v_t at d = 64, C = 16."""
    x = make(2, 2, 768, 64, seed=91)
    dS = ttt.ttt_assoc_state_fwd(x["K"], x["V"], x["eta"], C=16)
    _, Sr = orc.assoc_scan(np_(x["Q"]), np_(x["K"]), np_(x["V"]), eta_of(x), None,
                           threads=THREADS)
    assert max_rel_l2(dS, Sr, 2) <= TOL


def test_unsupported_shapes_raise_before_launch(cuda_lib):
    n0 = ttt.launch_count()
    x = make(1, 1, 96, 64, seed=3)      # T = 96: a multiple of C = 16 but not of 64
    with pytest.raises(ttt.TTTError) as e:
        ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], x["eta"], None, C=16)
    assert e.value.status == 2
    x = make(1, 1, 128, 32, seed=4)     # head dim 32
    with pytest.raises(ttt.TTTError) as e:
        ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], x["eta"], None, C=64)
    assert e.value.status == 2
    assert ttt.launch_count() == n0
