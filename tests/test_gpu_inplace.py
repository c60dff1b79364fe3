"""GPU parity of inplace_ttt_chunk_fwd against the fp64 oracle, through the C ABI.

Tolerance: relative L2 error <= 1e-2 (bf16 inputs) for O and for the final W, taken per output
column (each column of O and W depends only on the same column of Vhat and W0).
"""
import numpy as np
import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu
TOL = 1e-2


def run(x, C, **kw):
    return ttt.inplace_ttt_chunk_fwd(x["Z"], x["Vhat"], x["W0"], x["eta"], C=C, **kw)


def check(x, C, O, W, cols=None):
    Z = x["Z"].float().cpu().numpy()
    Or, Wr = orc.inplace_chunks(Z, x["Vhat"].float().cpu().numpy(),
                                x["W0"].float().cpu().numpy(), x["eta"], C, cols=cols)
    if cols is not None:
        O, W = O[:, cols], W[:, cols]
    eo = max_rel_l2(O.t().contiguous(), Or.T, 1)
    ew = max_rel_l2(W.t().contiguous(), Wr.T, 1)
    assert eo <= TOL and ew <= TOL, (eo, ew)
    return eo, ew


@pytest.mark.parametrize("T,C,Dff,D", [
    (128, 128, 128, 64),     # one chunk
    (256, 128, 128, 64),
    (384, 128, 256, 128),
    (512, 256, 384, 256),
    (768, 256, 256, 320),    # D not a multiple of 128: 64-wide tiles
    (640, 128, 640, 512),
])
def test_small_shapes(cuda_lib, T, C, Dff, D):
    x = inp.inplace_inputs(T, Dff, D, seed=T + Dff + D, device="cuda", eta=1e-2)
    O, W = run(x, C)
    check(x, C, O, W)
    assert ttt.read_device_error() == 0


def test_full_wdown_workload_column_subset(cuda_lib):
    w = inp.WORKLOADS["inplace_bf16_T32768_Dff9728_D2560_C1024"]
    x = inp.make_inputs(w, "cuda")
    O, W = run(x, w.C)
    cols = np.arange(3, w.D, 20)  # every 20th column: each is exact on its own
    eo, ew = check(x, w.C, O, W, cols=cols)
    print(f"in-place W_down workload ({len(cols)} of {w.D} columns): max rel L2 O {eo:.2e} "
          f"W {ew:.2e}")
    assert torch.isfinite(O.float()).all() and torch.isfinite(W).all()
    assert ttt.read_device_error() == 0


def test_zero_eta_keeps_W0_and_reads_it_every_chunk(cuda_lib):
    x = inp.inplace_inputs(384, 256, 128, seed=2, device="cuda", eta=0.0)
    O, W = run(x, 128)
    assert torch.equal(W, x["W0"].float())
    ref = (x["Z"].double() @ x["W0"].double())
    assert max_rel_l2(O.t().contiguous(), ref.t().contiguous(), 1) < TOL


def test_one_launch_per_chunk_and_determinism(cuda_lib):
    x = inp.inplace_inputs(512, 256, 256, seed=4, device="cuda", eta=1e-2)
    n0 = ttt.launch_count()
    O1, W1 = run(x, 128)
    assert ttt.launch_count() - n0 == 4
    O2, W2 = run(x, 128)
    assert torch.equal(O1, O2) and torch.equal(W1, W2)


def test_workspace_and_shape_errors(cuda_lib):
    x = inp.inplace_inputs(256, 128, 64, seed=5, device="cuda")
    small = torch.empty(16, device="cuda", dtype=torch.uint8)
    with pytest.raises(ttt.TTTError) as e:
        run(x, 128, workspace=small)
    assert e.value.status == 3
    with pytest.raises(ttt.TTTError) as e:
        run(x, 64)  # C not a multiple of 128
    assert e.value.status == 2


@pytest.mark.parametrize("T,C,Dff,D", [
    (512, 256, 256, 256),     # one chunk pair
    (768, 256, 512, 512),     # a pair, then a single chunk
    (2048, 512, 384, 768),    # two pairs
])
def test_chunk_pairs_match_oracle_and_single_chunks(cuda_lib, tuning, T, C, Dff, D):
    """Two chunks per launch (chunk i+1's read corrected by eta (Z_(i+1) Z_i^T) Vhat_i, one
    update over both chunks) against the oracle, and against one chunk per launch."""
    x = inp.inplace_inputs(T, Dff, D, seed=T + C + D, device="cuda", eta=1e-2)
    n0 = ttt.launch_count()
    O2, W2 = run(x, C)
    n_pairs = (T // C) // 2
    assert ttt.launch_count() - n0 == T // C - n_pairs
    check(x, C, O2, W2)
    tuning("inplace_chunks_per_launch", 1)
    O1, W1 = run(x, C)
    assert max_rel_l2(O2.t().contiguous(), O1.t().contiguous(), 1) < 1e-2
    assert max_rel_l2(W2.t().contiguous(), W1.t().contiguous(), 1) < 1e-4
    assert ttt.read_device_error() == 0
