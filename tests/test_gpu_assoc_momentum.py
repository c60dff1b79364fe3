"""GPU parity of ttt_assoc_momentum_fwd (associative mode with a momentum inner loop) against
the fp64 oracle's token-by-token momentum recurrence, through the C ABI: the one-pass form that
carries both states (the default; every beta in [0, 1]) and the two-pass plain + decayed form
(momentum_form 1; beta in [0.25, 0.9]). The oracle is pinned on the CPU (tests/test_oracle_pins.py:
beta = 0, closed weighted-sum forms including beta = 1, hand-worked tokens). Tolerance: per-(b,h)
relative L2 <= 1e-2 for O, S_out and M_out (bf16 inputs and outputs)."""
import os

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
    g = torch.Generator("cuda").manual_seed(seed + 3)
    x["S0"] = torch.randn(B, H, 128, 128, device="cuda", generator=g) * 0.05 if states else None
    x["M0"] = torch.randn(B, H, 128, 128, device="cuda", generator=g) * 0.05 if states else None
    return x


def run(x, beta, **kw):
    return ttt.ttt_assoc_momentum_fwd(x["Q"], x["K"], x["V"], x["eta"], beta, x["S0"], x["M0"],
                                      C=64, eta_scalar=x["eta_scalar"], **kw)


def check(x, beta, got, streams=None):
    eta = x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()
    f = lambda t: None if t is None else t.float().cpu().numpy()
    ref = orc.assoc_momentum(f(x["Q"]), f(x["K"]), f(x["V"]), eta, beta, f(x["S0"]), f(x["M0"]),
                             threads=os.cpu_count() or 4, streams=streams)
    errs = []
    for name, g, r in zip(("O", "S", "M"), got, ref):
        if streams is not None:
            g = torch.stack([g[b, h] for b, h in streams])
        e = max_rel_l2(g, r, 1 if streams is not None else 2)
        errs.append(e)
        assert e <= TOL, (name, e)
    return errs


BETAS = [0.0, 0.25, 0.5, 0.9, 0.99, 0.999, 1.0]


@pytest.mark.parametrize("beta", BETAS)
@pytest.mark.parametrize("B,H,T", [(1, 1, 64), (1, 2, 512), (2, 3, 640)])
def test_momentum_matches_oracle(cuda_lib, B, H, T, beta):
    x = make(B, H, T, seed=T + 7 * H + int(1000 * beta))
    check(x, beta, run(x, beta))
    assert ttt.read_device_error() == 0


@pytest.mark.parametrize("beta", [0.25, 0.5, 0.75, 0.9])
def test_two_pass_form_matches_oracle(cuda_lib, tuning, beta):
    """The plain + decayed evaluation, kept as a comparison variant, within its beta range."""
    tuning("momentum_form", 1)
    x = make(2, 3, 640, seed=11 + int(100 * beta))
    check(x, beta, run(x, beta))
    assert ttt.read_device_error() == 0


@pytest.mark.parametrize("beta", [0.9, 0.999])
@pytest.mark.parametrize("parts", ["1", "2", "4", "16"])
def test_forced_superchunk_counts(cuda_lib, tuning, parts, beta):
    """Split into superchunks (pass 1 maps the pieces, the scan composes them, pass 2 starts
    every part from its composed state), every split gives the oracle's results."""
    tuning("assoc_parts", int(parts))
    x = make(1, 2, 1024, seed=31)
    check(x, beta, run(x, beta))
    assert ttt.read_device_error() == 0


def test_forms_agree(cuda_lib, tuning):
    """Both forms evaluate the same recurrence: well inside the oracle tolerance of each other."""
    x = make(2, 2, 1024, seed=77)
    got = run(x, 0.8)
    tuning("momentum_form", 1)
    ref = run(x, 0.8)
    for g, r in zip(got, ref):
        assert max_rel_l2(g, r, 2) < 5e-3
    # deterministic: the default form gives the same bits again
    tuning("momentum_form", 0)
    again = run(x, 0.8)
    for g, r in zip(got, again):
        assert torch.equal(g, r)


def test_scalar_eta_zero_states_and_state_aliasing(cuda_lib):
    x = make(1, 2, 256, seed=4, eta="const", states=False)
    check(x, 0.8, run(x, 0.8))
    y = make(1, 2, 256, seed=5)
    O1, S1, M1 = run(y, 0.7)
    S_io, M_io = y["S0"].clone(), y["M0"].clone()
    y2 = dict(y, S0=S_io, M0=M_io)
    O2, S2, M2 = run(y2, 0.7, S_out=S_io, M_out=M_io)
    assert torch.equal(O1, O2) and torch.equal(S1, S2) and torch.equal(M1, M2)


def test_state_carry_across_calls(cuda_lib):
    """Momentum state (S, M) carried from the first half of a sequence into the second."""
    x = make(1, 1, 1024, seed=9)
    O, S, M = run(x, 0.9)
    half = {k: (v[:, :, :512].contiguous() if torch.is_tensor(v) and v.dim() == 4 and
                v.shape[2] == 1024 else v) for k, v in x.items()}
    rest = {k: (v[:, :, 512:].contiguous() if torch.is_tensor(v) and v.dim() == 4 and
                v.shape[2] == 1024 else v) for k, v in x.items()}
    for k in ("eta",):
        half[k] = x[k][:, :, :512].contiguous()
        rest[k] = x[k][:, :, 512:].contiguous()
    Oa, Sa, Ma = run(half, 0.9)
    rest["S0"], rest["M0"] = Sa, Ma
    Ob, Sb, Mb = run(rest, 0.9)
    assert max_rel_l2(torch.cat([Oa, Ob], dim=2), O, 2) < 1e-2
    assert max_rel_l2(Sb, S, 2) < 1e-2 and max_rel_l2(Mb, M, 2) < 1e-2


def test_full_associative_workload_sampled_streams(cuda_lib):
    w = inp.WORKLOADS["assoc_momentum_bf16_B4H16T65536_d128C64"]
    x = inp.make_inputs(w, "cuda")
    x["S0"], x["M0"] = None, None
    got = run(x, 0.99)
    streams = [(0, 0), (1, 7), (2, 9), (3, 15)]
    errs = check(x, 0.99, got, streams=streams)
    print("associative momentum (beta 0.99, 4 sampled streams): max rel L2 O %.2e S %.2e "
          "M %.2e" % tuple(errs))
    assert all(torch.isfinite(t).all() for t in got)
    assert ttt.read_device_error() == 0


def test_errors(cuda_lib, tuning):
    x = make(1, 1, 128, seed=1)
    for beta in (-0.1, 1.5, float("nan")):
        with pytest.raises(ttt.TTTError) as e:
            run(x, beta)
        assert e.value.status == 2
    tuning("momentum_form", 1)
    for beta in (0.0, 0.1, 0.95, 1.0):
        with pytest.raises(ttt.TTTError) as e:
            run(x, beta)
        assert e.value.status == 2
    tuning("momentum_form", 0)
    with pytest.raises(ttt.TTTError) as e:
        run(x, 0.5, workspace=torch.empty(16, device="cuda", dtype=torch.uint8))
    assert e.value.status == 3
