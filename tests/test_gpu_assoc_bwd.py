"""GPU parity of ttt_assoc_scan_bwd (backward of the associative mode) against the fp64 oracle's
adjoint sweep, through the C ABI. The oracle's backward is pinned on the CPU to central finite
differences and to autograd (tests/test_oracle_pins.py). Tolerance: per-(b,h) relative L2
<= 1e-2 for dQ, dK, dV, deta and dS0 (bf16 inputs and outputs)."""
import os

import numpy as np
import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu
TOL = 1e-2


def make(B, H, T, seed, eta="sigmoid", states=True):
    x = inp.dual_or_assoc_inputs(B, H, T, 128, seed=seed, device="cuda", normalise=("Q", "K"),
                                 eta=eta, eta_const=0.25, w0="zero")
    g = torch.Generator("cuda").manual_seed(seed + 1)
    x["dO"] = torch.randn(B, H, T, 128, device="cuda", generator=g).to(torch.bfloat16)
    x["S0"] = (torch.randn(B, H, 128, 128, device="cuda", generator=g) * 0.05) if states else None
    x["dS_out"] = (torch.randn(B, H, 128, 128, device="cuda", generator=g) * 0.05
                   if states else None)
    return x


def run(x, **kw):
    return ttt.ttt_assoc_scan_bwd(x["Q"], x["K"], x["V"], x["eta"], x["S0"], x["dO"],
                                  x["dS_out"], C=64, eta_scalar=x["eta_scalar"], **kw)


def check(x, got, streams=None):
    eta = x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()
    f = lambda t: None if t is None else t.float().cpu().numpy()
    ref = orc.assoc_scan_bwd(f(x["Q"]), f(x["K"]), f(x["V"]), eta, f(x["S0"]), f(x["dO"]),
                             f(x["dS_out"]), threads=os.cpu_count() or 4, streams=streams)
    errs = []
    for name, g, r in zip(("dQ", "dK", "dV", "deta", "dS0"), got, ref):
        if streams is not None:
            g = torch.stack([g[b, h] for b, h in streams])
        e = max_rel_l2(g, r, 1 if streams is not None else 2)
        errs.append(e)
        assert e <= TOL, (name, e)
    return errs


@pytest.mark.parametrize("B,H,T", [(1, 1, 64), (1, 2, 256), (2, 3, 640), (1, 1, 4096)])
def test_small_shapes(cuda_lib, B, H, T):
    x = make(B, H, T, seed=T + 11 * B + H)
    check(x, run(x))
    assert ttt.read_device_error() == 0


def test_scalar_eta_and_zero_states(cuda_lib):
    x = make(1, 2, 512, seed=3, eta="const", states=False)
    assert x["eta"] is None
    check(x, run(x))


def test_zero_and_tiny_rates(cuda_lib):
    """Rows whose rate is zero or tiny get the oracle's dV and deta like every other row; a zero
    scalar rate gives exactly zero dK and dV."""
    x = make(1, 2, 512, seed=21)
    x["eta"][:, :, ::7] = 0.0
    x["eta"][:, :, 3::11] = 1e-30
    check(x, run(x))
    x = make(1, 1, 256, seed=22, eta="const", states=False)
    x["eta_scalar"] = 0.0
    got = run(x)
    assert torch.count_nonzero(got[2]) == 0 and torch.count_nonzero(got[1]) == 0
    check(x, got)


@pytest.mark.parametrize("parts", ["1", "2", "4", "16"])
def test_forced_superchunk_counts(cuda_lib, tuning, parts):
    """The reverse-order passes split into superchunks give the oracle's gradients for every P."""
    tuning("assoc_parts", int(parts))
    x = make(1, 2, 1024, seed=77)
    check(x, run(x))


def test_deterministic_and_caller_buffers(cuda_lib):
    x = make(1, 2, 256, seed=8)
    a = run(x)
    bufs = dict(dQ=torch.empty_like(x["Q"]), dK=torch.empty_like(x["Q"]),
                dV=torch.empty_like(x["Q"]), deta=torch.empty(1, 2, 256, device="cuda"),
                dS0=torch.empty(1, 2, 128, 128, device="cuda"))
    b = run(x, **bufs)
    for u, v, w in zip(a, b, bufs.values()):
        assert torch.equal(u, v) and v.data_ptr() == w.data_ptr()


def test_full_associative_workload_sampled_streams(cuda_lib):
    w = inp.WORKLOADS["assoc_bf16_B4H16T65536_d128C64"]
    x = inp.make_inputs(w, "cuda")
    g = torch.Generator("cuda").manual_seed(99)
    x["dO"] = torch.randn(x["Q"].shape, device="cuda", generator=g).to(torch.bfloat16)
    x["S0"] = None
    x["dS_out"] = torch.randn(4, 16, 128, 128, device="cuda", generator=g) * 0.05
    got = run(x)
    errs = check(x, got, streams=[(0, 0), (3, 15)])
    print("associative backward (2 sampled streams): max rel L2 dQ %.2e dK %.2e dV %.2e "
          "deta %.2e dS0 %.2e" % tuple(errs))
    assert all(torch.isfinite(t.float()).all() for t in got)
    assert ttt.read_device_error() == 0


def test_errors(cuda_lib):
    x96 = make(1, 1, 96, seed=1)   # T = 96: a multiple of C = 32 but not of the 64-token tile
    with pytest.raises(ttt.TTTError) as e:
        ttt.ttt_assoc_scan_bwd(x96["Q"], x96["K"], x96["V"], x96["eta"], None, x96["dO"], C=32)
    assert e.value.status == 2
    x = make(1, 1, 128, seed=1)
    with pytest.raises(ttt.TTTError) as e:
        run(x, workspace=torch.empty(16, device="cuda", dtype=torch.uint8))
    assert e.value.status == 3
    with pytest.raises(ttt.TTTError) as e:    # an output aliasing an input
        run(x, dQ=x["dO"])
    assert e.value.status == 1


@pytest.mark.parametrize("parts", [1, 2, 4])
def test_separate_and_fused_reverse_passes(cuda_lib, tuning, parts):
    """dV and dK from the two separate reverse passes (assoc_bwd_form 1) and from the fused one
    that carries the state gradient once (the default) both meet the oracle for every superchunk
    split, and agree well inside its tolerance."""
    tuning("assoc_parts", parts)
    x = make(1, 3, 1024, seed=41 + parts)
    fused = run(x)
    check(x, fused)
    tuning("assoc_bwd_form", 1)
    separate = run(x)
    check(x, separate)
    for g, r in zip(fused, separate):
        assert max_rel_l2(g, r, 2) < 5e-3
    assert ttt.read_device_error() == 0
