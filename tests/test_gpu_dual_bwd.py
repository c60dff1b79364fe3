"""GPU parity of ttt_linear_dual_bwd (backward of the TTT-Linear dual form) against the fp64
oracle's chunk-wise adjoint, through the C ABI. The oracle's backward is pinned on the CPU to
central finite differences and to autograd through mini-batch steps (tests/test_oracle_pins.py).
Tolerance: per-(b,h) relative L2 <= 1e-2 for dQ, dK, dV, deta and dW0 (bf16 inputs/outputs)."""
import os

import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu
TOL = 1e-2
C = 16


def make(B, H, T, d, seed, eta="sigmoid", states=True):
    x = inp.dual_or_assoc_inputs(B, H, T, d, seed=seed, device="cuda", normalise=("K", "V"),
                                 eta=eta, eta_const=0.3, w0="normal_0.02")
    g = torch.Generator("cuda").manual_seed(seed + 1)
    x["dO"] = torch.randn(B, H, T, d, device="cuda", generator=g).to(torch.bfloat16)
    x["dW_out"] = (torch.randn(B, H, d, d, device="cuda", generator=g) * 0.05
                   if states else None)
    if not states:
        x["W0"] = None
    return x


def run(x, **kw):
    return ttt.ttt_linear_dual_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"], x["dO"],
                                   x["dW_out"], C=C, eta_scalar=x["eta_scalar"], **kw)


def check(x, got, streams=None):
    eta = x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()
    f = lambda t: None if t is None else t.float().cpu().numpy()
    ref = orc.dual_form_bwd(f(x["Q"]), f(x["K"]), f(x["V"]), eta, f(x["W0"]), f(x["dO"]),
                            f(x["dW_out"]), C, threads=os.cpu_count() or 4, streams=streams)
    errs = []
    for name, g, r in zip(("dQ", "dK", "dV", "deta", "dW0"), got, ref):
        if streams is not None:
            g = torch.stack([g[b, h] for b, h in streams])
        e = max_rel_l2(g, r, 1 if streams is not None else 2)
        errs.append(e)
        assert e <= TOL, (name, e)
    return errs


@pytest.mark.parametrize("B,H,T,d", [(1, 1, 16, 64), (1, 2, 256, 64), (2, 3, 640, 64),
                                     (1, 2, 272, 32), (1, 2, 208, 128)])
def test_small_shapes(cuda_lib, B, H, T, d):
    """Rates sigmoid(z) (up to 1: the state moves a lot per chunk), random W0 and dW_out."""
    x = make(B, H, T, d, seed=T + 11 * B + H + d)
    check(x, run(x))
    assert ttt.read_device_error() == 0


def test_scalar_eta_and_zero_states(cuda_lib):
    x = make(1, 2, 512, 64, seed=3, eta="const", states=False)
    assert x["eta"] is None
    check(x, run(x))


@pytest.mark.parametrize("T", [272, 1024])
def test_zero_and_tiny_rates(cuda_lib, T):
    """Per-token rates of exactly zero and of 1e-25 mixed with ordinary ones, in the same 16-token
    chunk, in the same 128-token stage and alone in whole stages; then every rate zero (the
    states never move, dV = 0, deta = -G . (A'^T dO + K X) still nonzero). The stage form takes
    deta from G itself wherever a rate is too small to divide by."""
    x = make(1, 2, T, 64, seed=T + 71)
    eta = x["eta"].clone()
    eta[0, 0, 3] = 0.0
    eta[0, 0, 5] = 1e-25
    eta[0, 0, 140:150] = 0.0
    eta[0, 1, 128:256] = 0.0
    eta[0, 1, 17] = 1e-25
    x["eta"] = eta
    check(x, run(x))
    x["eta"] = torch.zeros_like(eta)
    got = run(x)
    check(x, got)
    assert float(got[2].float().abs().max()) == 0.0   # dV = -dG = 0
    assert float(got[3].abs().max()) > 0.0            # deta does not vanish with the rates
    assert ttt.read_device_error() == 0


def test_deterministic_and_caller_buffers(cuda_lib):
    x = make(1, 2, 256, 64, seed=8)
    a = run(x)
    bufs = dict(dQ=torch.empty_like(x["Q"]), dK=torch.empty_like(x["Q"]),
                dV=torch.empty_like(x["Q"]), deta=torch.empty(1, 2, 256, device="cuda"),
                dW0=torch.empty(1, 2, 64, 64, device="cuda"))
    b = run(x, **bufs)
    for u, v, w in zip(a, b, bufs.values()):
        assert torch.equal(u, v) and v.data_ptr() == w.data_ptr()


def _workload_case(name, seed):
    w = inp.WORKLOADS[name]
    x = inp.make_inputs(w, "cuda")
    g = torch.Generator("cuda").manual_seed(seed)
    x["dO"] = torch.randn(x["Q"].shape, device="cuda", generator=g).to(torch.bfloat16)
    x["dW_out"] = torch.randn(w.B, w.H, w.d, w.d, device="cuda", generator=g) * 0.05
    return x


def test_125m_layer_workload_all_streams(cuda_lib):
    """B=8, H=12, T=2048, d=64 with the forward workload's distributions; every stream."""
    x = _workload_case("dual_bf16_B8H12T2048_d64C16", 5)
    errs = check(x, run(x))
    print("dual backward, B8 H12 T2048 (all streams): max rel L2 dQ %.2e dK %.2e dV %.2e "
          "deta %.2e dW0 %.2e" % tuple(errs))


def test_long_context_workload_sampled_streams(cuda_lib):
    """B=2, H=32, T=32768, d=64: two sampled streams against the oracle."""
    x = _workload_case("dual_bf16_B2H32T32768_d64C16", 6)
    got = run(x)
    errs = check(x, got, streams=[(0, 0), (1, 31)])
    print("dual backward, B2 H32 T32768 (2 sampled streams): max rel L2 dQ %.2e dK %.2e "
          "dV %.2e deta %.2e dW0 %.2e" % tuple(errs))
    assert all(torch.isfinite(t.float()).all() for t in got)
    assert ttt.read_device_error() == 0


def test_errors(cuda_lib):
    x = make(1, 1, 128, 64, seed=1)
    with pytest.raises(ttt.TTTError) as e:      # only C = 16 is supported
        ttt.ttt_linear_dual_bwd(x["Q"], x["K"], x["V"], x["eta"], None, x["dO"], C=32)
    assert e.value.status == 2
    with pytest.raises(ttt.TTTError) as e:
        run(x, workspace=torch.empty(16, device="cuda", dtype=torch.uint8))
    assert e.value.status == 3
    with pytest.raises(ttt.TTTError) as e:      # an output aliasing an input
        run(x, dQ=x["dO"])
    assert e.value.status == 1
    y = make(1, 1, 128, 48, seed=2)
    with pytest.raises(ttt.TTTError) as e:
        run(y)
    assert e.value.status == 2


@pytest.mark.parametrize("T", [16, 272, 1024])
def test_backward_forms_agree(cuda_lib, tuning, T):
    """d = 64: the stage form (the default), the one-kernel form with its own forward sweep
    (dual_bwd_form 1) and the reverse sweep on the stage kernel's chunk checkpoints (2) all give
    the oracle's gradients, full and partial 128-token stages included."""
    x = make(2, 2, T, 64, seed=T + 5)
    a = run(x)
    check(x, a)
    for form in (1, 2):
        tuning("dual_bwd_form", form)
        b = run(x)
        check(x, b)
        # The forms round different operands to bf16 (the stage form: -diag(eta) G, W_s, dG and
        # the masked stage scores; the others: G and every chunk-start W), each within the
        # oracle's 1e-2 bar on its own, so they agree to within that bar, not tighter.
        for g, r in zip(a, b):
            assert max_rel_l2(g, r, 2) < 1e-2
    assert ttt.read_device_error() == 0
