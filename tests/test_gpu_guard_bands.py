"""Guard bands around every output (GPU): each entry point writes into outputs that sit inside
larger buffers whose 4 KB before and after hold a canary byte; after the call the canaries must
be unchanged (compute-sanitizer is closed on this machine; this catches a kernel writing past an
output, e.g. in a ragged last tile). Shapes with ragged tails where the kernels have them."""
import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from _helpers import guarded, guards_intact
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu


def _check(*pairs):
    torch.cuda.synchronize()
    for i, (view, buf) in enumerate(pairs):
        assert guards_intact(view, buf), i
    assert ttt.read_device_error() == 0


def test_dual_forward_bf16_and_fp32(cuda_lib):
    # 13 chunks: a full 8-chunk stage and a partial one; 3 streams split over CTA pairs
    x = inp.dual_or_assoc_inputs(1, 3, 208, 64, seed=1, device="cuda", normalise=("K", "V"))
    O = guarded((1, 3, 208, 64), torch.bfloat16, "cuda")
    W = guarded((1, 3, 64, 64), torch.float32, "cuda")
    ttt.ttt_linear_dual_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"], C=16, O=O[0], W_out=W[0])
    _check(O, W)
    x = inp.dual_or_assoc_inputs(1, 2, 80, 32, seed=2, device="cuda", dtype="f32",
                                 qkv="normal_1_over_d", eta="const", eta_const=0.1, w0="zero")
    O = guarded((1, 2, 80, 32), torch.float32, "cuda")
    W = guarded((1, 2, 32, 32), torch.float32, "cuda")
    ttt.ttt_linear_dual_fwd(x["Q"], x["K"], x["V"], None, None, C=16, eta_scalar=0.1, O=O[0],
                            W_out=W[0])
    _check(O, W)


def test_dual_segmented_forward_and_backwards(cuda_lib):
    x = inp.dual_or_assoc_inputs(1, 1, 1024, 64, seed=3, device="cuda", normalise=("K", "V"))
    O = guarded((1, 1, 1024, 64), torch.bfloat16, "cuda")
    W = guarded((1, 1, 64, 64), torch.float32, "cuda")
    ttt.ttt_linear_dual_seg_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"], C=16, segments=4,
                                O=O[0], W_out=W[0])
    _check(O, W)
    g = torch.Generator("cuda").manual_seed(4)
    dO = torch.randn(1, 1, 1024, 64, device="cuda", generator=g).to(torch.bfloat16)
    for fn, kw in ((ttt.ttt_linear_dual_bwd, {}), (ttt.ttt_linear_dual_seg_bwd, {"segments": 4})):
        outs = [guarded((1, 1, 1024, 64), torch.bfloat16, "cuda") for _ in range(3)]
        de = guarded((1, 1, 1024), torch.float32, "cuda")
        dW = guarded((1, 1, 64, 64), torch.float32, "cuda")
        fn(x["Q"], x["K"], x["V"], x["eta"], x["W0"], dO, None, C=16, dQ=outs[0][0],
           dK=outs[1][0], dV=outs[2][0], deta=de[0], dW0=dW[0], **kw)
        _check(*outs, de, dW)


def test_associative_forward_momentum_and_backward(cuda_lib):
    x = inp.dual_or_assoc_inputs(1, 2, 192, 128, seed=5, device="cuda", normalise=("Q", "K"),
                                 eta="sigmoid", w0="zero")
    O = guarded((1, 2, 192, 128), torch.bfloat16, "cuda")
    S = guarded((1, 2, 128, 128), torch.float32, "cuda")
    ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], x["eta"], None, C=64, O=O[0], S_out=S[0])
    _check(O, S)
    O = guarded((1, 2, 192, 128), torch.bfloat16, "cuda")
    S = guarded((1, 2, 128, 128), torch.float32, "cuda")
    M = guarded((1, 2, 128, 128), torch.float32, "cuda")
    ttt.ttt_assoc_momentum_fwd(x["Q"], x["K"], x["V"], x["eta"], 0.5, None, None, C=64, O=O[0],
                               S_out=S[0], M_out=M[0])
    _check(O, S, M)
    g = torch.Generator("cuda").manual_seed(6)
    dO = torch.randn(1, 2, 192, 128, device="cuda", generator=g).to(torch.bfloat16)
    outs = [guarded((1, 2, 192, 128), torch.bfloat16, "cuda") for _ in range(3)]
    de = guarded((1, 2, 192), torch.float32, "cuda")
    dS = guarded((1, 2, 128, 128), torch.float32, "cuda")
    ttt.ttt_assoc_scan_bwd(x["Q"], x["K"], x["V"], x["eta"], None, dO, None, C=64,
                           dQ=outs[0][0], dK=outs[1][0], dV=outs[2][0], deta=de[0], dS0=dS[0])
    _check(*outs, de, dS)


def test_inplace_update_and_lm_target(cuda_lib):
    # D = 320: 64-wide tiles at the edge of the 256-wide ones
    x = inp.inplace_inputs(768, 256, 320, seed=7, device="cuda", eta=1e-2)
    O = guarded((768, 320), torch.bfloat16, "cuda")
    W = guarded((256, 320), torch.float32, "cuda")
    ttt.inplace_ttt_chunk_fwd(x["Z"], x["Vhat"], x["W0"], x["eta"], C=256, O=O[0], W_out=W[0])
    _check(O, W)
    y = inp.inplace_lm_inputs(512, 128, 320, 384, 3, seed=8, device="cuda")
    V = guarded((512, 320), torch.bfloat16, "cuda")
    ttt.ttt_lm_target_fwd(y["X"], y["Wc"], y["Wp"], Vhat=V[0])
    _check(V)
