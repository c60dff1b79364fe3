"""GPU parity of ttt_linear_dual_fwd against the fp64 oracle, through the C ABI.

Tolerances (max over (b,h) slices of the relative L2 error, for O and for the final W):
1e-4 for fp32 inputs, 1e-2 for bf16 inputs.
"""
import os

import numpy as np
import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import f64, max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-4, "bf16": 1e-2}


def run(x, C, **kw):
    return ttt.ttt_linear_dual_fwd(x["Q"], x["K"], x["V"], x["eta"], x.get("W0"), C=C,
                                   eta_scalar=x["eta_scalar"], **kw)


def oracle(x, C, streams=None):
    eta = x["eta_scalar"] if x["eta"] is None else x["eta"].cpu().numpy()
    W0 = None if x.get("W0") is None else x["W0"].cpu().numpy()
    Q, K, V = (x[k].float().cpu().numpy() for k in ("Q", "K", "V"))
    return orc.dual_form(Q, K, V, eta, W0, C, threads=os.cpu_count() or 4, streams=streams)


def check(x, C, O, W, tol, streams=None):
    Or, Wr = oracle(x, C, streams)
    if streams is not None:
        O = torch.stack([O[b, h] for b, h in streams])
        W = torch.stack([W[b, h] for b, h in streams])
        lead = 1
    else:
        lead = 2
    eo, ew = max_rel_l2(O, Or, lead), max_rel_l2(W, Wr, lead)
    assert eo <= tol and ew <= tol, (eo, ew)
    return eo, ew


def workload(name, **over):
    w = inp.WORKLOADS[name]
    return w, inp.make_inputs(w, "cuda", **over)


def test_fp32_tiny_workload(cuda_lib):
    w, x = workload("dual_f32_B1H2T256_d32C16")
    O, W = run(x, w.C)
    check(x, w.C, O, W, TOL["f32"])
    # W0 given as NULL (zeros) gives the same bits as an explicit zero tensor
    x0 = dict(x, W0=None)
    O0, W0_ = run(x0, w.C)
    assert torch.equal(O, O0) and torch.equal(W, W0_)
    assert ttt.read_device_error() == 0


def test_bf16_125m_layer_workload(cuda_lib):
    w, x = workload("dual_bf16_B8H12T2048_d64C16")
    O, W = run(x, w.C)
    eo, ew = check(x, w.C, O, W, TOL["bf16"])
    print(f"dual 125M-layer workload: max rel L2 O {eo:.2e} W {ew:.2e}")
    assert ttt.read_device_error() == 0


def test_bf16_long_context_workload(cuda_lib):
    """Every stream of the 1.3B-layer long-context shape against the oracle, one batch item at a
    time (32 streams per oracle call keeps the host memory small)."""
    w, x = workload("dual_bf16_B2H32T32768_d64C16")
    O, W = run(x, w.C)
    worst = (0.0, 0.0)
    for b in range(w.B):
        sub = {k: (v[b:b + 1] if torch.is_tensor(v) else v) for k, v in x.items()}
        eo, ew = check(sub, w.C, O[b:b + 1], W[b:b + 1], TOL["bf16"])
        worst = (max(worst[0], eo), max(worst[1], ew))
    print(f"dual long-context workload (all {w.B * w.H} streams): max rel L2 O {worst[0]:.2e} "
          f"W {worst[1]:.2e}")
    assert ttt.read_device_error() == 0


SWEEP = [(d, C, m, B, H) for d in (32, 64, 128) for C in (1, 16, 64) for m in (1, 2, 7)
         for (B, H) in ((1, 1), (1, 3), (3, 1)) if (d + C + m + B) % 3 == 0 or C == 16]


@pytest.mark.parametrize("d,C,m,B,H", SWEEP)
def test_sweep_bf16(cuda_lib, d, C, m, B, H):
    x = inp.dual_or_assoc_inputs(B, H, m * C, d, seed=d * 1000 + C * 10 + m, device="cuda",
                                 normalise=("K", "V"))
    O, W = run(x, C)
    check(x, C, O, W, TOL["bf16"])


@pytest.mark.parametrize("d,C,m", [(32, 16, 3), (64, 1, 5), (64, 64, 2), (128, 16, 2)])
def test_sweep_fp32(cuda_lib, d, C, m):
    x = inp.dual_or_assoc_inputs(2, 2, m * C, d, seed=7 + d + C, device="cuda", dtype="f32",
                                 qkv="normal_1_over_d", eta="sigmoid_over_d")
    O, W = run(x, C)
    check(x, C, O, W, TOL["f32"])


@pytest.mark.parametrize("T", [16, 48, 64, 80, 112, 128, 272, 1040])
def test_ragged_stage_tails(cuda_lib, T):
    """T that is not a multiple of the kernels' pipeline stages (partial last stage)."""
    x = inp.dual_or_assoc_inputs(2, 3, T, 64, seed=T, device="cuda", normalise=("K", "V"))
    O, W = run(x, 16)
    check(x, 16, O, W, TOL["bf16"])


def test_state_aliasing_W_out_equals_W0(cuda_lib):
    x = inp.dual_or_assoc_inputs(2, 2, 256, 64, seed=3, device="cuda", normalise=("K", "V"))
    O_ref, W_ref = run(x, 16)
    W_io = x["W0"].clone()
    O, W = ttt.ttt_linear_dual_fwd(x["Q"], x["K"], x["V"], x["eta"], W_io, C=16, W_out=W_io)
    assert W.data_ptr() == W_io.data_ptr()
    assert torch.equal(O, O_ref) and torch.equal(W_io, W_ref)


def test_determinism_permutation_and_state_carry(cuda_lib):
    x = inp.dual_or_assoc_inputs(2, 3, 512, 64, seed=11, device="cuda", normalise=("K", "V"))
    O1, W1 = run(x, 16)
    O2, W2 = run(x, 16)
    assert torch.equal(O1, O2) and torch.equal(W1, W2)  # bitwise run-to-run
    # batch items are independent: permuting streams permutes outputs, bit for bit
    perm = torch.tensor([4, 0, 5, 2, 1, 3], device="cuda")
    xp = {k: (v.reshape(6, *v.shape[2:])[perm].reshape(v.shape) if torch.is_tensor(v) else v)
          for k, v in x.items()}
    Op, Wp = run(xp, 16)
    assert torch.equal(Op.reshape(6, 512, 64), O1.reshape(6, 512, 64)[perm])
    assert torch.equal(Wp.reshape(6, 64, 64), W1.reshape(6, 64, 64)[perm])
    # state carry: two calls over the halves, chained through W_out -> W0, equal one call. The
    # chain is the same arithmetic wherever the split falls (W bit-identical); the outputs of the
    # d = 64 kernel are formed per 128-token stage, so they are bit-identical for a split on a
    # stage boundary and equal within rounding for a split inside a stage.
    for h, exact_o in ((256, True), (208, False)):
        xa = {k: (v[:, :, :h].contiguous() if torch.is_tensor(v) and v.dim() >= 3 and k != "W0"
                  else v) for k, v in x.items()}
        xb = {k: (v[:, :, h:].contiguous() if torch.is_tensor(v) and v.dim() >= 3 and k != "W0"
                  else v) for k, v in x.items()}
        Oa, Wa = run(xa, 16)
        xb["W0"] = Wa
        Ob, Wb = run(xb, 16)
        assert torch.equal(Wb, W1)
        Ocat = torch.cat([Oa, Ob], dim=2)
        if exact_o:
            assert torch.equal(Ocat, O1)
        else:
            assert max_rel_l2(Ocat, O1, 2) < 5e-3


def test_column_split_variants_agree_bitwise(cuda_lib, tuning):
    """The all-warp-MMA kernels compute every column the same way whether a stream sits on one
    CTA or is split over two."""
    tuning("dual_kernel", 1)
    for d, T in ((64, 256), (128, 128)):
        x = inp.dual_or_assoc_inputs(1, 4, T, d, seed=d, device="cuda", normalise=("K", "V"))
        outs = []
        for split in (1, 2):
            tuning("dual_column_split", split)
            outs.append(run(x, 16))
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("warp_cols", [16, 8])
def test_tensor_core_form_column_splits(cuda_lib, tuning, warp_cols):
    """The stage-form kernel (chain on warp MMAs, outputs on tcgen05) with 1, 2 and 4 CTAs per
    stream and 16 or 8 columns per chain warp: the chain of a column is the same arithmetic in
    every split (final W bit-identical), and every split meets the oracle on full and partial
    128-token stages."""
    tuning("dual_kernel", 3)
    tuning("dual_warp_cols", warp_cols)
    for T in (16, 144, 400):
        x = inp.dual_or_assoc_inputs(2, 3, T, 64, seed=T + 11, device="cuda",
                                     normalise=("K", "V"))
        outs = []
        for split in (1, 2, 4):
            tuning("dual_column_split", split)
            O, W = run(x, 16)
            check(x, 16, O, W, TOL["bf16"])
            outs.append((O, W))
        for O, W in outs[1:]:
            assert torch.equal(W, outs[0][1])
            assert max_rel_l2(O, outs[0][0], 2) < 1e-3
        assert ttt.read_device_error() == 0


@pytest.mark.parametrize("warp_cols", [16, 8])
def test_tensor_core_and_warp_forms_agree(cuda_lib, tuning, warp_cols):
    """The stage form regroups the output sum (the earlier chunks of a stage enter through the
    masked scores instead of the chunk-start state); the chain is the same as the all-warp-MMA
    kernel's with as many columns per warp, so W agrees bit for bit and O within the bf16
    rounding of the regrouped terms."""
    x = inp.dual_or_assoc_inputs(2, 4, 1024, 64, seed=31, device="cuda", normalise=("K", "V"))
    tuning("dual_warp_cols", warp_cols)
    tuning("dual_kernel", 1)
    Ow, Ww = run(x, 16)
    tuning("dual_kernel", 3)
    Ot, Wt = run(x, 16)
    assert torch.equal(Ww, Wt)
    assert max_rel_l2(Ot, Ow, 2) < 5e-3


def test_degenerate_cases(cuda_lib):
    # eta = 0: no update; O = Q W0
    x = inp.dual_or_assoc_inputs(1, 2, 128, 64, seed=9, device="cuda", normalise=("K", "V"),
                                 eta="const", eta_const=0.0)
    O, W = run(x, 16)
    assert torch.equal(W, x["W0"])
    check(x, 16, O, W, TOL["bf16"])
    # keys all zero: residual is -V but the update K^T G vanishes; O = Q W0
    x["K"] = torch.zeros_like(x["K"])
    x["eta"], x["eta_scalar"] = None, 0.5
    O, W = run(x, 16)
    assert torch.equal(W, x["W0"])
    check(x, 16, O, W, TOL["bf16"])


def test_one_launch_per_call(cuda_lib):
    x = inp.dual_or_assoc_inputs(1, 1, 64, 64, seed=1, device="cuda")
    n0 = ttt.launch_count()
    run(x, 16)
    run(x, 4)
    assert ttt.launch_count() - n0 == 2


def test_invalid_calls_raise_before_launch(cuda_lib):
    x = inp.dual_or_assoc_inputs(1, 1, 64, 64, seed=1, device="cuda")
    n0 = ttt.launch_count()
    with pytest.raises(ttt.TTTError) as e:
        run(x, 24)  # T % C != 0
    assert e.value.status == 1
    x48 = inp.dual_or_assoc_inputs(1, 1, 64, 48, seed=1, device="cuda")
    with pytest.raises(ttt.TTTError) as e:
        run(x48, 16)
    assert e.value.status == 2
    assert ttt.launch_count() == n0


@pytest.mark.parametrize("form", [1, 2])
@pytest.mark.parametrize("warp_cols", [8, 16])
@pytest.mark.parametrize("split", [1, 2])
def test_kernel_variants_match_oracle(cuda_lib, tuning, warp_cols, split, form):
    """Every all-warp-MMA variant (8 or 16 output columns per warp, one or two CTAs per stream,
    chain and outputs on one warp or on a warp pair) meets the bf16 tolerance on full and partial
    pipeline stages."""
    if form == 2 and warp_cols == 8:
        pytest.skip("the warp-pair form exists for 16-column warps")
    tuning("dual_warp_cols", warp_cols)
    tuning("dual_column_split", split)
    tuning("dual_kernel", form)
    for T in (144, 512):
        x = inp.dual_or_assoc_inputs(2, 3, T, 64, seed=T + 3, device="cuda", normalise=("K", "V"))
        O, W = run(x, 16)
        check(x, 16, O, W, TOL["bf16"])


def test_pair_and_single_forms_agree_bitwise(cuda_lib, tuning):
    """The warp-pair form performs the single-warp form's arithmetic in the same order."""
    x = inp.dual_or_assoc_inputs(2, 3, 400, 64, seed=21, device="cuda", normalise=("K", "V"))
    for split in (1, 2):
        tuning("dual_column_split", split)
        outs = []
        for form in (1, 2):
            tuning("dual_kernel", form)
            outs.append(run(x, 16))
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("C,T", [(32, 32), (32, 96), (32, 416), (64, 64), (64, 192), (64, 576)])
def test_tensor_core_form_larger_chunks(cuda_lib, tuning, C, T):
    """C = 32 and 64 on the stage kernel (one gradient step per C tokens: the chunk's residuals
    all at the chunk-start W), with 1, 2 and 4 CTAs per stream, full and partial stages."""
    x = inp.dual_or_assoc_inputs(2, 3, T, 64, seed=C * 100 + T, device="cuda",
                                 normalise=("K", "V"))
    for split in (1, 2, 4):
        tuning("dual_column_split", split)
        O, W = run(x, C)
        check(x, C, O, W, TOL["bf16"])
    assert ttt.read_device_error() == 0


def test_split_form_matches_oracle_and_stage_kernel(cuda_lib, tuning):
    """Chain CTAs and output CTAs on separate SMs of one cluster (stages handed over by
    distributed-shared-memory copies), with one or two streams per cluster (also an odd stream
    count: the last cluster holds one): every case meets the oracle on full and partial stages
    and its final state equals the single-SM stage kernel's bit for bit (the same chain)."""
    for B, H, T in ((2, 3, 16), (2, 3, 144), (1, 5, 1040)):
        x = inp.dual_or_assoc_inputs(B, H, T, 64, seed=T + 71 + H, device="cuda",
                                     normalise=("K", "V"))
        tuning("dual_kernel", 3)
        tuning("dual_column_split", 1)
        O_tc, W_tc = run(x, 16)
        tuning("dual_column_split", 0)
        tuning("dual_kernel", 4)
        for ks in (1, 2):
            tuning("dual_cluster_streams", ks)
            n0 = ttt.launch_count()
            O, W = run(x, 16)
            assert ttt.launch_count() - n0 == 1
            check(x, 16, O, W, TOL["bf16"])
            assert torch.equal(W, W_tc)
            assert max_rel_l2(O, O_tc, 2) < 1e-3
        assert ttt.read_device_error() == 0
