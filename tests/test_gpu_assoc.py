"""GPU parity of ttt_assoc_scan_fwd against the fp64 oracle, through the C ABI.

The oracle's chunked form is used for speed; it is pinned to the sequential recurrence on the CPU
(tests/test_oracle_pins.py). Tolerance: per-(b,h) relative L2 <= 1e-2 for O and the final S.
"""
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


def make(B, H, T, seed, **kw):
    return inp.dual_or_assoc_inputs(B, H, T, 128, seed=seed, device="cuda",
                                    normalise=("Q", "K"), eta=kw.pop("eta", "sigmoid"),
                                    w0=kw.pop("w0", "zero"), **kw)


def run(x, S0=None, **kw):
    return ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], x["eta"], S0, C=64,
                                  eta_scalar=x["eta_scalar"], **kw)


def check(x, O, S, S0=None, streams=None):
    eta = x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()
    Q, K, V = (x[k].float().cpu().numpy() for k in ("Q", "K", "V"))
    s0 = None if S0 is None else S0.cpu().numpy()
    Or, Sr = orc.assoc_scan(Q, K, V, eta, s0, form="chunked", C=64,
                            threads=os.cpu_count() or 4, streams=streams)
    if streams is not None:
        O = torch.stack([O[b, h] for b, h in streams])
        S = torch.stack([S[b, h] for b, h in streams])
        lead = 1
    else:
        lead = 2
    eo, es = max_rel_l2(O, Or, lead), max_rel_l2(S, Sr, lead)
    assert eo <= TOL and es <= TOL, (eo, es)
    return eo, es


@pytest.mark.parametrize("B,H,T", [(1, 1, 64), (1, 2, 128), (1, 1, 1024), (2, 3, 640),
                                   (1, 1, 4096)])
def test_small_shapes_default_parts(cuda_lib, B, H, T):
    x = make(B, H, T, seed=T + B + H)
    O, S = run(x)
    check(x, O, S)
    assert ttt.read_device_error() == 0


@pytest.mark.parametrize("parts", ["1", "2", "4", "16"])
def test_forced_superchunk_counts_agree(cuda_lib, tuning, parts):
    """The two-pass prefix scan over P superchunks gives the oracle's result for every P."""
    tuning("assoc_parts", int(parts))
    x = make(1, 2, 1024, seed=77)
    S0 = torch.randn(1, 2, 128, 128, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    n0 = ttt.launch_count()
    O, S = run(x, S0)
    assert ttt.launch_count() - n0 == (1 if parts == "1" else 3)
    eo, es = check(x, O, S, S0)
    assert eo <= RACE_TRIPWIRE and es <= RACE_TRIPWIRE, (eo, es)


# The kernel's own error on these inputs is bf16 rounding of Q, K, eta*V, the bf16 state copy and
# the score tile: about 3e-3 for O and 2e-3 for S. A chunk that reads a stale or half-written
# operand (a synchronisation fault between the warp groups) raises it well above that while
# often staying under the 1e-2 parity bar, so these cases also check a bound of twice the level.
RACE_TRIPWIRE = 6e-3


def test_full_associative_workload_every_stream(cuda_lib):
    """Every stream of the full associative workload against the oracle, one batch item (16
    streams, both superchunks of each) per oracle call."""
    w = inp.WORKLOADS["assoc_bf16_B4H16T65536_d128C64"]
    x = inp.make_inputs(w, "cuda")
    O, S = run(x)
    worst = (0.0, 0.0)
    for b in range(w.B):
        sub = {k: (v[b:b + 1] if torch.is_tensor(v) else v) for k, v in x.items()}
        eo, es = check(sub, O[b:b + 1], S[b:b + 1])
        worst = (max(worst[0], eo), max(worst[1], es))
    print(f"associative workload (all {w.B * w.H} streams): max rel L2 O {worst[0]:.2e} "
          f"S {worst[1]:.2e}")
    assert worst[0] <= RACE_TRIPWIRE and worst[1] <= RACE_TRIPWIRE, worst
    assert ttt.read_device_error() == 0


def test_scalar_eta_aliasing_and_determinism(cuda_lib):
    x = make(1, 2, 512, seed=5, eta="const", eta_const=0.25)
    S0 = torch.randn(1, 2, 128, 128, device="cuda") * 0.1
    O1, S1 = run(x, S0)
    check(x, O1, S1, S0)
    O2, S2 = run(x, S0)
    assert torch.equal(O1, O2) and torch.equal(S1, S2)
    Sio = S0.clone()
    O3, S3 = run(x, Sio, S_out=Sio)
    assert torch.equal(O3, O1) and torch.equal(Sio, S1)


def test_state_carry_across_calls(cuda_lib):
    x = make(1, 1, 1024, seed=9)
    O, S = run(x)
    half = {k: (v[:, :, :512].contiguous() if torch.is_tensor(v) and v.dim() >= 3 else v)
            for k, v in x.items()}
    rest = {k: (v[:, :, 512:].contiguous() if torch.is_tensor(v) and v.dim() >= 3 else v)
            for k, v in x.items()}
    Oa, Sa = run(half)
    Ob, Sb = run(rest, Sa)
    assert max_rel_l2(torch.cat([Oa, Ob], dim=2), O, 2) < 1e-2
    assert max_rel_l2(Sb, S, 2) < 1e-2


def test_errors(cuda_lib):
    x = make(1, 1, 96, seed=1)   # T = 96: a multiple of C = 32 but not of the 64-token tile
    with pytest.raises(ttt.TTTError) as e:
        ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], x["eta"], None, C=32)
    assert e.value.status == 2
    xs = make(1, 1, 1024, seed=2)
    lib = ttt.load_library()
    need = lib.ttt_assoc_scan_workspace_size(1, 1, 1024, 128, 64, 1)
    assert need > 0  # one stream splits into several superchunks
    with pytest.raises(ttt.TTTError) as e:
        run(xs, workspace=torch.empty(16, device="cuda", dtype=torch.uint8))
    assert e.value.status == 3
