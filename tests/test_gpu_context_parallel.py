"""GPU checks of the context-parallel pieces, through the C ABI: for the associative scan the
slice state increment, the prefix combination of increments, a sequence split into slices
evaluated slice by slice (the ranks emulated one after another in one process: no kernel waits
on another), and the orchestrator on a one-rank NCCL group; for the dual form the slice maps,
their ordered fold and the slices run from the folded starts."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import max_rel_l2
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200 import inputs as inp
from weight_linear_attention_ttt_b200.shard import split_range

pytestmark = pytest.mark.gpu
TOL = 1e-2


def make(B, H, T, seed):
    return inp.dual_or_assoc_inputs(B, H, T, 128, seed=seed, device="cuda", normalise=("Q", "K"),
                                    eta="sigmoid", w0="normal_0.02")


def oracle_full(x, S0):
    return orc.assoc_scan(x["Q"].float().cpu().numpy(), x["K"].float().cpu().numpy(),
                          x["V"].float().cpu().numpy(), x["eta"].cpu().numpy(),
                          None if S0 is None else S0.cpu().numpy(), form="chunked", C=64,
                          threads=os.cpu_count() or 4)


def test_state_increment_matches_oracle(cuda_lib):
    x = make(2, 3, 640, seed=31)
    dS = ttt.ttt_assoc_state_fwd(x["K"], x["V"], x["eta"], C=64)
    _, ref = oracle_full(x, None)
    assert max_rel_l2(dS, ref, 2) <= TOL
    # scalar learning rate
    dS2 = ttt.ttt_assoc_state_fwd(x["K"], x["V"], None, C=64, eta_scalar=0.5)
    _, ref2 = orc.assoc_scan(x["Q"].float().cpu().numpy(), x["K"].float().cpu().numpy(),
                             x["V"].float().cpu().numpy(), 0.5, None, form="chunked", C=64)
    assert max_rel_l2(dS2, ref2, 2) <= TOL


def test_prefix_sum_of_increments(cuda_lib):
    g = torch.Generator("cuda").manual_seed(5)
    inc = torch.randn(4, 2, 3, 128, 128, device="cuda", generator=g)
    S0 = torch.randn(2, 3, 128, 128, device="cuda", generator=g)
    for upto in range(5):
        out = ttt.ttt_state_prefix_sum(S0, inc, upto)
        ref = S0.double() + inc[:upto].double().sum(0)
        assert torch.allclose(out.double(), ref, rtol=1e-6, atol=1e-5)
    out = ttt.ttt_state_prefix_sum(None, inc, 2)
    assert torch.allclose(out, inc[0] + inc[1])


@pytest.mark.parametrize("ranks", [2, 3, 5])
def test_sequence_split_into_slices_equals_one_pass(cuda_lib, ranks):
    B, H, T = 2, 2, 64 * 15
    x = make(B, H, T, seed=40 + ranks)
    S0 = torch.randn(B, H, 128, 128, device="cuda") * 0.05
    spans = [split_range(T // 64, r, ranks) for r in range(ranks)]
    sl = [{k: (v[:, :, 64 * a:64 * b].contiguous() if torch.is_tensor(v) and v.dim() >= 3 and
               k != "W0" else v) for k, v in x.items()} for a, b in spans]
    inc = torch.stack([ttt.ttt_assoc_state_fwd(s["K"], s["V"], s["eta"], C=64) for s in sl])
    outs = []
    for r, s in enumerate(sl):
        start = ttt.ttt_state_prefix_sum(S0, inc, r)
        O, _ = ttt.ttt_assoc_scan_fwd(s["Q"], s["K"], s["V"], s["eta"], start, C=64)
        outs.append(O)
    S_final = ttt.ttt_state_prefix_sum(S0, inc, ranks)
    Or, Sr = oracle_full(x, S0)
    assert max_rel_l2(torch.cat(outs, dim=2), Or, 2) <= TOL
    assert max_rel_l2(S_final, Sr, 2) <= TOL


def test_orchestrator_on_a_one_rank_nccl_group(cuda_lib):
    import torch.distributed as dist

    from weight_linear_attention_ttt_b200.context_parallel import assoc_scan_fwd_cp

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x = make(1, 2, 512, seed=50)
        S0 = torch.randn(1, 2, 128, 128, device="cuda") * 0.05
        O, S = assoc_scan_fwd_cp(x["Q"], x["K"], x["V"], x["eta"], S0, C=64)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    Or, Sr = oracle_full(x, S0)
    assert max_rel_l2(O, Or, 2) <= TOL and max_rel_l2(S, Sr, 2) <= TOL


def test_dual_form_orchestrator_on_a_one_rank_nccl_group(cuda_lib):
    import torch.distributed as dist

    from weight_linear_attention_ttt_b200.context_parallel import dual_form_fwd_cp

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x = inp.dual_or_assoc_inputs(1, 2, 512, 64, seed=51, device="cuda",
                                     normalise=("K", "V"), eta="sigmoid")
        O, W = dual_form_fwd_cp(x["Q"], x["K"], x["V"], x["eta"], x["W0"], C=16)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    f = lambda t: t.float().cpu().numpy()
    Or, Wr = orc.dual_form(f(x["Q"]), f(x["K"]), f(x["V"]), x["eta"].cpu().numpy(),
                           x["W0"].cpu().numpy(), 16)
    assert max_rel_l2(O, Or, 2) <= TOL and max_rel_l2(W, Wr, 2) <= TOL


@pytest.mark.parametrize("slices,dtype", [(2, "bf16"), (4, "bf16"), (3, "f32")])
def test_dual_form_slices_emulated_on_one_gpu(cuda_lib, slices, dtype):
    """The dual form's context-parallel pieces on one GPU: every slice's affine maps
    (ttt_linear_dual_slice_maps), the ordered fold of the maps before it
    (ttt_dual_state_fold) as its start state, and the dual form on the slice from there; the
    concatenated outputs and the fold of all maps equal the sequential oracle."""
    import torch

    B, H, T, d, C = 2, 2, 768 if slices == 3 else 1024, 32 if dtype == "f32" else 64, 16
    x = inp.dual_or_assoc_inputs(B, H, T, d, seed=40 + slices, device="cuda", dtype=dtype,
                                 normalise=("K", "V"), eta="sigmoid")
    L = T // slices
    cut = lambda t, r: t[:, :, r * L:(r + 1) * L].contiguous()
    maps = [ttt.ttt_linear_dual_slice_maps(cut(x["K"], r), cut(x["V"], r), cut(x["eta"], r),
                                           C=C) for r in range(slices)]
    A_all = torch.stack([m[0] for m in maps]).contiguous()
    B_all = torch.stack([m[1] for m in maps]).contiguous()
    outs = []
    for r in range(slices):
        start = ttt.ttt_dual_state_fold(x["W0"], A_all, B_all, r)
        O_r, _ = ttt.ttt_linear_dual_fwd(cut(x["Q"], r), cut(x["K"], r), cut(x["V"], r),
                                         cut(x["eta"], r), start, C=C)
        outs.append(O_r)
    W = ttt.ttt_dual_state_fold(x["W0"], A_all, B_all, slices)
    f = lambda t: t.float().cpu().numpy()
    Or, Wr = orc.dual_form(f(x["Q"]), f(x["K"]), f(x["V"]), x["eta"].cpu().numpy(),
                           x["W0"].cpu().numpy(), C)
    tol = 1e-4 if dtype == "f32" else 1e-2
    eo = max_rel_l2(torch.cat(outs, dim=2), Or, 2)
    ew = max_rel_l2(W, Wr, 2)
    assert eo <= tol and ew <= tol, (eo, ew)
    # fold of nothing is W0; W_out may be the W0 buffer
    assert torch.equal(ttt.ttt_dual_state_fold(x["W0"], A_all, B_all, 0), x["W0"])
    W0c = x["W0"].clone()
    ttt.ttt_dual_state_fold(W0c, A_all, B_all, slices, W_out=W0c)
    assert torch.equal(W0c, W)
    assert ttt.read_device_error() == 0
