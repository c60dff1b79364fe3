"""GPU parity of ttt_linear_dual_seg_fwd (the dual form evaluated sequence-parallel by the
segment-affine scan) against the fp64 oracle's sequential chunk loop, through the C ABI. The
oracle's own segmented evaluation is pinned to the sequential loop on the CPU
(tests/test_oracle_pins.py). Tolerances as for the dual form: per-(b,h) relative L2 <= 1e-2 for
bf16 inputs and 1e-4 for fp32 inputs, O and W_out."""
import os

import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu


def check(x, C, O, W, tol, streams=None):
    eta = x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()
    W0 = None if x.get("W0") is None else x["W0"].cpu().numpy()
    Q, K, V = (x[k].float().cpu().numpy() for k in ("Q", "K", "V"))
    Or, Wr = orc.dual_form(Q, K, V, eta, W0, C, threads=os.cpu_count() or 4, streams=streams)
    if streams is not None:
        O = torch.stack([O[b, h] for b, h in streams])
        W = torch.stack([W[b, h] for b, h in streams])
    lead = 1 if streams is not None else 2
    eo, ew = max_rel_l2(O, Or, lead), max_rel_l2(W, Wr, lead)
    assert eo <= tol and ew <= tol, (eo, ew)
    return eo, ew


def run(x, C, segments, **kw):
    return ttt.ttt_linear_dual_seg_fwd(x["Q"], x["K"], x["V"], x["eta"], x.get("W0"), C=C,
                                       segments=segments, eta_scalar=x["eta_scalar"], **kw)


@pytest.mark.parametrize("B,H,T,d,S", [(1, 1, 1024, 64, 4), (1, 2, 2048, 64, 8),
                                       (2, 1, 4096, 64, 0), (1, 2, 1024, 32, 16),
                                       (1, 1, 1024, 128, 4), (1, 1, 512, 64, 32)])
def test_bf16_against_the_sequential_oracle(cuda_lib, B, H, T, d, S):
    x = inp.dual_or_assoc_inputs(B, H, T, d, seed=T + d + S, device="cuda",
                                 normalise=("K", "V"))
    O, W = run(x, 16, S)
    check(x, 16, O, W, 1e-2)
    assert ttt.read_device_error() == 0


def test_fp32_against_the_sequential_oracle(cuda_lib):
    x = inp.dual_or_assoc_inputs(1, 2, 1024, 32, seed=9, device="cuda", dtype="f32",
                                 qkv="normal_1_over_d", eta="const", eta_const=0.1, w0="zero")
    O, W = run(x, 16, 8)
    check(x, 16, O, W, 1e-4)


def test_strong_rates_and_state_aliasing(cuda_lib):
    """Rates up to 1 (each segment map contracts strongly); W_out may be the W0 buffer."""
    x = inp.dual_or_assoc_inputs(1, 2, 2048, 64, seed=12, device="cuda", normalise=("K", "V"),
                                 eta="sigmoid")
    O, W = run(x, 16, 8)
    check(x, 16, O, W, 1e-2)
    W0 = x["W0"].clone()
    O2, W2 = run(x, 16, 8, W_out=x["W0"])
    assert W2.data_ptr() == x["W0"].data_ptr()
    assert torch.equal(O2, O) and torch.equal(W2, W)
    x["W0"].copy_(W0)


def test_automatic_choice_with_many_streams_is_the_sequential_kernel(cuda_lib):
    """With B*H streams filling the GPU the automatic count is 1: the same bits as
    ttt_linear_dual_fwd."""
    x = inp.dual_or_assoc_inputs(8, 12, 256, 64, seed=4, device="cuda", normalise=("K", "V"))
    lib = ttt.load_library()
    assert lib.ttt_linear_dual_seg_workspace_size(8, 12, 256, 64, 16, 1, 0) == 0
    O, W = run(x, 16, 0)
    O1, W1 = ttt.ttt_linear_dual_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"], C=16)
    assert torch.equal(O, O1) and torch.equal(W, W1)


def test_few_streams_long_sequence_workload(cuda_lib):
    """B=1, H=4, T=262144, d=64 (the workload the segmented evaluation is for), every stream."""
    w = inp.WORKLOADS["dual_seg_bf16_B1H4T262144_d64C16"]
    x = inp.make_inputs(w, "cuda")
    O, W = run(x, 16, 0)
    eo, ew = check(x, 16, O, W, 1e-2)
    print("segmented dual form, B1 H4 T262144 (all streams): max rel L2 O %.2e W %.2e"
          % (eo, ew))
    assert ttt.read_device_error() == 0


def test_errors(cuda_lib):
    x = inp.dual_or_assoc_inputs(1, 1, 1024, 64, seed=1, device="cuda", normalise=("K", "V"))
    with pytest.raises(ttt.TTTError) as e:     # 3 does not divide the 64 chunks
        run(x, 16, 3)
    assert e.value.status == 1
    with pytest.raises(ttt.TTTError) as e:
        run(x, 16, 4, workspace=torch.empty(16, device="cuda", dtype=torch.uint8))
    assert e.value.status == 3


def _bwd_case(B, H, T, d, seed, eta="sigmoid"):
    x = inp.dual_or_assoc_inputs(B, H, T, d, seed=seed, device="cuda", normalise=("K", "V"),
                                 eta=eta, eta_const=0.3)
    g = torch.Generator("cuda").manual_seed(seed + 1)
    x["dO"] = torch.randn(B, H, T, d, device="cuda", generator=g).to(torch.bfloat16)
    x["dW_out"] = torch.randn(B, H, d, d, device="cuda", generator=g) * 0.05
    return x


def check_bwd(x, got, streams=None):
    eta = x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()
    f = lambda t: None if t is None else t.float().cpu().numpy()
    ref = orc.dual_form_bwd(f(x["Q"]), f(x["K"]), f(x["V"]), eta, f(x["W0"]), f(x["dO"]),
                            f(x["dW_out"]), 16, threads=os.cpu_count() or 4, streams=streams)
    errs = []
    for name, g, r in zip(("dQ", "dK", "dV", "deta", "dW0"), got, ref):
        if streams is not None:
            g = torch.stack([g[b, h] for b, h in streams])
        e = max_rel_l2(g, r, 1 if streams is not None else 2)
        errs.append(e)
        assert e <= 1e-2, (name, e)
    return errs


def run_bwd(x, segments, **kw):
    return ttt.ttt_linear_dual_seg_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"], x["dO"],
                                       x["dW_out"], C=16, segments=segments,
                                       eta_scalar=x["eta_scalar"], **kw)


@pytest.mark.parametrize("B,H,T,d,S", [(1, 1, 1024, 64, 4), (1, 2, 2048, 64, 8),
                                       (2, 1, 1024, 64, 0), (1, 2, 1024, 32, 16),
                                       (1, 1, 512, 128, 4)])
def test_backward_against_the_sequential_oracle(cuda_lib, B, H, T, d, S):
    x = _bwd_case(B, H, T, d, seed=T + d + S + 3)
    check_bwd(x, run_bwd(x, S))
    assert ttt.read_device_error() == 0


def test_backward_scalar_rate_and_zero_states(cuda_lib):
    x = _bwd_case(1, 2, 1024, 64, seed=31, eta="const")
    x["W0"], x["dW_out"] = None, None
    check_bwd(x, run_bwd(x, 8))


def test_backward_few_streams_long_sequence(cuda_lib):
    """B=1, H=4, T=262144, d=64: every stream against the sequential oracle backward."""
    w = inp.WORKLOADS["dual_seg_bwd_bf16_B1H4T262144_d64C16"]
    x = inp.make_inputs(w, "cuda")
    errs = check_bwd(x, run_bwd(x, 0))
    print("segmented dual backward, B1 H4 T262144 (all streams): max rel L2 dQ %.2e dK %.2e "
          "dV %.2e deta %.2e dW0 %.2e" % tuple(errs))
    assert ttt.read_device_error() == 0


def test_backward_errors(cuda_lib):
    x = _bwd_case(1, 1, 1024, 64, seed=2)
    with pytest.raises(ttt.TTTError) as e:     # 3 does not divide the 64 chunks
        run_bwd(x, 3)
    assert e.value.status == 1
    with pytest.raises(ttt.TTTError) as e:
        run_bwd(x, 4, workspace=torch.empty(16, device="cuda", dtype=torch.uint8))
    assert e.value.status == 3
