"""torch.autograd wrappers: the layer's forward and backward as one differentiable call.

Outer-loop training differentiates through the inner updates ("RNN의 기억을 작은 모델로 바꾼다면:
Test-Time Training 읽기", mini-batch section; "KV 바인딩 기반 테스트 시간 학습은 사실상 선형
어텐션이다": the layer is trained end to end). Each wrapper's forward calls the library's forward
entry point and its backward calls the matching backward entry point; the wrappers only route
tensors (argument marshalling, like the rest of the binding): every product runs in the
library's kernels.

    O, W_out = ttt_dual_linear(Q, K, V, eta, W0, C=16)     # gradients for Q, K, V, eta, W0
    O, S_out = ttt_assoc_scan(Q, K, V, eta, S0, C=64)      # gradients for Q, K, V, eta, S0

eta may be None (then eta_scalar is used and gets no gradient); W0 / S0 may be None (zeros, no
gradient). The backwards support what ttt_linear_dual_bwd / ttt_assoc_scan_bwd support (bf16,
dual form C = 16, associative mode d = 128, C = 64).
"""
from __future__ import annotations

import sys

import torch


def _lib():
    """The binding package, looked up at call time."""
    return sys.modules[__package__]


def _grad_or_zeros(g, like):
    return torch.zeros_like(like) if g is None else g.contiguous()


class _DualLinear(torch.autograd.Function):
    @staticmethod
    def forward(ctx, Q, K, V, eta, W0, C, eta_scalar):
        O, W_out = _lib().ttt_linear_dual_fwd(Q, K, V, eta, W0, C=C, eta_scalar=eta_scalar)
        ctx.save_for_backward(Q, K, V, eta, W0)
        ctx.C, ctx.eta_scalar = C, eta_scalar
        ctx.has_eta, ctx.has_w0 = eta is not None, W0 is not None
        return O, W_out

    @staticmethod
    def backward(ctx, dO, dW_out):
        Q, K, V, eta, W0 = ctx.saved_tensors
        dQ, dK, dV, deta, dW0 = _lib().ttt_linear_dual_bwd(
            Q, K, V, eta, W0, _grad_or_zeros(dO, Q),
            None if dW_out is None else dW_out.contiguous(), C=ctx.C,
            eta_scalar=ctx.eta_scalar)
        return (dQ, dK, dV, deta if ctx.has_eta else None, dW0 if ctx.has_w0 else None, None,
                None)


class _AssocScan(torch.autograd.Function):
    @staticmethod
    def forward(ctx, Q, K, V, eta, S0, C, eta_scalar):
        O, S_out = _lib().ttt_assoc_scan_fwd(Q, K, V, eta, S0, C=C, eta_scalar=eta_scalar)
        ctx.save_for_backward(Q, K, V, eta, S0)
        ctx.C, ctx.eta_scalar = C, eta_scalar
        ctx.has_eta, ctx.has_s0 = eta is not None, S0 is not None
        return O, S_out

    @staticmethod
    def backward(ctx, dO, dS_out):
        Q, K, V, eta, S0 = ctx.saved_tensors
        dQ, dK, dV, deta, dS0 = _lib().ttt_assoc_scan_bwd(
            Q, K, V, eta, S0, _grad_or_zeros(dO, Q),
            None if dS_out is None else dS_out.contiguous(), C=ctx.C,
            eta_scalar=ctx.eta_scalar)
        return (dQ, dK, dV, deta if ctx.has_eta else None, dS0 if ctx.has_s0 else None, None,
                None)


def ttt_dual_linear(Q, K, V, eta=None, W0=None, *, C: int, eta_scalar: float = 0.0):
    """Differentiable TTT-Linear dual form. Returns (O, W_out)."""
    return _DualLinear.apply(Q, K, V, eta, W0, C, eta_scalar)


def ttt_assoc_scan(Q, K, V, eta=None, S0=None, *, C: int, eta_scalar: float = 0.0):
    """Differentiable associative (gradient-ascent linear-attention) mode. Returns (O, S_out)."""
    return _AssocScan.apply(Q, K, V, eta, S0, C, eta_scalar)
