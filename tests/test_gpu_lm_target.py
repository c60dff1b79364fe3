"""GPU parity of the LM-aligned In-Place target (ttt_lm_target_fwd) and of the In-Place update
formed behind it (inplace_ttt_lm_chunk_fwd) against the fp64 oracle, through the C ABI. The
oracle's target is pinned on the CPU (tests/test_oracle_pins.py: brute-force loops, single taps,
causality). Tolerance: relative L2 <= 1e-2 per output column (bf16 inputs and outputs)."""
import numpy as np
import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu
TOL = 1e-2


def f64(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("T,Dm,D,k", [(128, 128, 64, 1), (256, 256, 128, 4), (512, 384, 320, 3),
                                      (384, 128, 256, 8)])
def test_target_matches_oracle(cuda_lib, T, Dm, D, k):
    x = inp.inplace_lm_inputs(T, 128, D, Dm, k, seed=T + Dm + D + k, device="cuda")
    V = ttt.ttt_lm_target_fwd(x["X"], x["Wc"], x["Wp"])
    ref = orc.lm_target(f64(x["X"]), f64(x["Wc"]), f64(x["Wp"]))
    assert max_rel_l2(V.t().contiguous(), ref.T, 1) <= TOL
    assert ttt.read_device_error() == 0


def test_target_reaches_exactly_one_token_ahead(cuda_lib):
    """Changing token 200 moves the targets of tokens 199 .. 199 + k - 1 only."""
    T, Dm, D, k = 256, 128, 64, 4
    x = inp.inplace_lm_inputs(T, 128, D, Dm, k, seed=3, device="cuda")
    V1 = ttt.ttt_lm_target_fwd(x["X"], x["Wc"], x["Wp"]).float()
    X2 = x["X"].clone()
    X2[200] += 4.0
    V2 = ttt.ttt_lm_target_fwd(X2, x["Wc"], x["Wp"]).float()
    moved = (V2 - V1).abs().amax(dim=1) > 0
    assert torch.equal(torch.nonzero(moved).flatten().cpu(), torch.arange(199, 199 + k))


@pytest.mark.parametrize("T,C,Dff,D,Dm", [(256, 128, 128, 64, 128), (512, 128, 256, 128, 256),
                                          (512, 256, 384, 256, 256)])
def test_update_with_lm_target_matches_oracle(cuda_lib, T, C, Dff, D, Dm):
    x = inp.inplace_lm_inputs(T, Dff, D, Dm, 4, seed=T + Dff, device="cuda", eta=1e-2)
    O, W = ttt.inplace_ttt_lm_chunk_fwd(x["Z"], x["X"], x["Wc"], x["Wp"], x["W0"], x["eta"], C=C)
    Vh = orc.lm_target(f64(x["X"]), f64(x["Wc"]), f64(x["Wp"]))
    Or, Wr = orc.inplace_chunks(f64(x["Z"]), Vh, f64(x["W0"]), x["eta"], C)
    assert max_rel_l2(O.t().contiguous(), Or.T, 1) <= TOL
    assert max_rel_l2(W.t().contiguous(), Wr.T, 1) <= TOL


def test_full_workload_column_subset(cuda_lib):
    w = inp.WORKLOADS["inplace_lm_bf16_T32768_Dff9728_D2560_Dm2560_C1024"]
    x = inp.make_inputs(w, "cuda")
    O, W = ttt.inplace_ttt_lm_chunk_fwd(x["Z"], x["X"], x["Wc"], x["Wp"], x["W0"], x["eta"],
                                        C=w.C)
    cols = np.arange(5, w.D, 160)
    Vh = orc.lm_target(f64(x["X"]), f64(x["Wc"]), f64(x["Wp"])[:, cols])
    Or, Wr = orc.inplace_chunks(f64(x["Z"]), Vh, f64(x["W0"])[:, cols], x["eta"], w.C)
    eo = max_rel_l2(O[:, cols].t().contiguous(), Or.T, 1)
    ew = max_rel_l2(W[:, cols].t().contiguous(), Wr.T, 1)
    print(f"in-place with LM target ({len(cols)} of {w.D} columns): max rel L2 O {eo:.2e} "
          f"W {ew:.2e}")
    assert eo <= TOL and ew <= TOL
    assert ttt.read_device_error() == 0


def test_errors(cuda_lib):
    x = inp.inplace_lm_inputs(128, 128, 64, 128, 4, seed=1, device="cuda")
    with pytest.raises(ttt.TTTError) as e:    # k > 8
        ttt.ttt_lm_target_fwd(x["X"], torch.zeros(9, 128, device="cuda"), x["Wp"])
    assert e.value.status == 2
    with pytest.raises(ttt.TTTError) as e:
        ttt.ttt_lm_target_fwd(x["X"], x["Wc"], x["Wp"],
                              workspace=torch.empty(16, device="cuda", dtype=torch.uint8))
    assert e.value.status == 3
