"""The torch.autograd wrappers route tensors to the right forward and backward entry points and
return each gradient to its own input (CPU: the library calls are replaced by fp64 oracle
stand-ins with the same signatures; the reference gradients come from torch autograd of
independent restatements of the forwards)."""
import numpy as np
import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from oracle import ttt_oracle as orc
from weight_linear_attention_ttt_b200.autograd import ttt_assoc_scan, ttt_dual_linear

B, H, T, d = 1, 2, 12, 3


def _np(t):
    return None if t is None else t.detach().numpy()


def _eta(eta, eta_scalar):
    return eta_scalar if eta is None else _np(eta)


def fake_dual_fwd(Q, K, V, eta, W0, *, C, eta_scalar=0.0):
    O, W = orc.dual_form(_np(Q), _np(K), _np(V), _eta(eta, eta_scalar), _np(W0), C)
    return torch.tensor(O), torch.tensor(W)


def fake_dual_bwd(Q, K, V, eta, W0, dO, dW_out=None, *, C, eta_scalar=0.0):
    out = orc.dual_form_bwd(_np(Q), _np(K), _np(V), _eta(eta, eta_scalar), _np(W0), _np(dO),
                            _np(dW_out), C)
    return tuple(torch.tensor(o) for o in out)


def fake_assoc_fwd(Q, K, V, eta, S0, *, C, eta_scalar=0.0):
    O, S = orc.assoc_scan(_np(Q), _np(K), _np(V), _eta(eta, eta_scalar), _np(S0))
    return torch.tensor(O), torch.tensor(S)


def fake_assoc_bwd(Q, K, V, eta, S0, dO, dS_out=None, *, C, eta_scalar=0.0):
    out = orc.assoc_scan_bwd(_np(Q), _np(K), _np(V), _eta(eta, eta_scalar), _np(S0), _np(dO),
                             _np(dS_out))
    return tuple(torch.tensor(o) for o in out)


@pytest.fixture
def fakes(monkeypatch):
    monkeypatch.setattr(ttt, "ttt_linear_dual_fwd", fake_dual_fwd)
    monkeypatch.setattr(ttt, "ttt_linear_dual_bwd", fake_dual_bwd)
    monkeypatch.setattr(ttt, "ttt_assoc_scan_fwd", fake_assoc_fwd)
    monkeypatch.setattr(ttt, "ttt_assoc_scan_bwd", fake_assoc_bwd)


def _inputs(seed, per_token, with_state):
    g = torch.Generator().manual_seed(seed)
    Q, K, V = (torch.randn(B, H, T, d, generator=g, dtype=torch.float64) * 0.6
               for _ in range(3))
    eta = (torch.rand(B, H, T, generator=g, dtype=torch.float64) * 0.4 + 0.05
           if per_token else None)
    W0 = torch.randn(B, H, d, d, generator=g, dtype=torch.float64) * 0.3 if with_state else None
    return Q, K, V, eta, W0


def _dual_reference(Q, K, V, eta, eta_scalar, W0, C):
    """Mini-batch TTT by definition, inner gradients by autograd (kept in the graph)."""
    O = torch.empty_like(Q)
    Ws = []
    for b in range(B):
        for h in range(H):
            W = torch.zeros(d, d, dtype=Q.dtype) if W0 is None else W0[b, h]
            outs = []
            for c0 in range(0, T, C):
                steps = []
                for s in range(c0, c0 + C):
                    Wr = W if W.requires_grad else W.detach().requires_grad_(True)
                    loss = 0.5 * ((K[b, h, s] @ Wr - V[b, h, s]) ** 2).sum()
                    (gW,) = torch.autograd.grad(loss, Wr, create_graph=True)
                    e = eta_scalar if eta is None else eta[b, h, s]
                    steps.append(e * gW)
                for t in range(c0, c0 + C):
                    outs.append(Q[b, h, t] @ (W - sum(steps[: t - c0 + 1])))
                W = W - sum(steps)
            O = O.index_put((torch.tensor([b]), torch.tensor([h])), torch.stack(outs)[None])
            Ws.append(W)
    return O, torch.stack(Ws).reshape(B, H, d, d)


@pytest.mark.parametrize("per_token,with_state,use_w", [(True, True, True), (False, False, True),
                                                       (True, False, False)])
def test_dual_wrapper_gradients(fakes, per_token, with_state, use_w):
    C = 4
    Q, K, V, eta, W0 = _inputs(3, per_token, with_state)
    leaves = [t for t in (Q, K, V, eta, W0) if t is not None]
    for t in leaves:
        t.requires_grad_(True)
    g = torch.Generator().manual_seed(9)
    R = torch.randn(B, H, T, d, generator=g, dtype=torch.float64)
    G = torch.randn(B, H, d, d, generator=g, dtype=torch.float64)
    O, W = ttt_dual_linear(Q, K, V, eta, W0, C=C, eta_scalar=0.2)
    L = (O * R).sum() + ((W * G).sum() if use_w else 0.0)
    grads = torch.autograd.grad(L, leaves)
    O2, W2 = _dual_reference(Q, K, V, eta, 0.2, W0, C)
    np.testing.assert_allclose(O.detach().numpy(), O2.detach().numpy(), rtol=1e-10, atol=1e-12)
    L2 = (O2 * R).sum() + ((W2 * G).sum() if use_w else 0.0)
    ref = torch.autograd.grad(L2, leaves)
    for a, r in zip(grads, ref):
        np.testing.assert_allclose(a.numpy(), r.numpy(), rtol=1e-8, atol=1e-10)


def _assoc_reference(Q, K, V, eta, eta_scalar, S0):
    O = []
    Ss = []
    for b in range(B):
        for h in range(H):
            S = torch.zeros(d, d, dtype=Q.dtype) if S0 is None else S0[b, h]
            outs = []
            for t in range(T):
                e = eta_scalar if eta is None else eta[b, h, t]
                S = S + e * torch.outer(K[b, h, t], V[b, h, t])
                outs.append(Q[b, h, t] @ S)
            O.append(torch.stack(outs))
            Ss.append(S)
    return torch.stack(O).reshape(B, H, T, d), torch.stack(Ss).reshape(B, H, d, d)


@pytest.mark.parametrize("per_token,with_state", [(True, True), (False, False)])
def test_assoc_wrapper_gradients(fakes, per_token, with_state):
    Q, K, V, eta, S0 = _inputs(5, per_token, with_state)
    leaves = [t for t in (Q, K, V, eta, S0) if t is not None]
    for t in leaves:
        t.requires_grad_(True)
    g = torch.Generator().manual_seed(11)
    R = torch.randn(B, H, T, d, generator=g, dtype=torch.float64)
    G = torch.randn(B, H, d, d, generator=g, dtype=torch.float64)
    O, S = ttt_assoc_scan(Q, K, V, eta, S0, C=4, eta_scalar=0.3)
    grads = torch.autograd.grad((O * R).sum() + (S * G).sum(), leaves)
    O2, S2 = _assoc_reference(Q, K, V, eta, 0.3, S0)
    ref = torch.autograd.grad((O2 * R).sum() + (S2 * G).sum(), leaves)
    for a, r in zip(grads, ref):
        np.testing.assert_allclose(a.numpy(), r.numpy(), rtol=1e-9, atol=1e-11)
