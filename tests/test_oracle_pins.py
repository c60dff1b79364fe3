"""Pins of the fp64 oracle to facts fixed by the pages and by the mathematics (CPU only).

Each test compares the oracle with something other than itself: gradients taken by autograd on
the inner loss (not the hand-derived gradient the oracle uses), closed forms, hand-worked
examples, or algebraically different forms of the same quantity. Sizes are tiny; fp64.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
rng = np.random.default_rng(7)


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ----------------------------------------------------------------------------- autograd helpers
def _grad_inner_loss(W: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
    """Gradient of the inner loss 1/2 ||k W - v||^2 at W, by autograd."""
    Wr = W.detach().clone().requires_grad_(True)
    loss = 0.5 * ((k @ Wr - v) ** 2).sum()
    (g,) = torch.autograd.grad(loss, Wr)
    return g


def _per_token_sgd(Q, K, V, eta, W0):
    """W_t = W_(t-1) - eta_t grad l(W_(t-1); x_t); o_t = q_t W_t (output from the updated model)."""
    Q, K, V, eta = (torch.as_tensor(x, dtype=torch.float64) for x in (Q, K, V, eta))
    W = torch.as_tensor(W0, dtype=torch.float64).clone()
    O = torch.empty_like(Q)
    for t in range(Q.shape[0]):
        W = W - eta[t] * _grad_inner_loss(W, K[t], V[t])
        O[t] = Q[t] @ W
    return O.numpy(), W.numpy()


def _minibatch_gd_by_definition(Q, K, V, eta, W0, C):
    """Mini-batch TTT: all gradients of a chunk are taken at the chunk-start weight W_b; token t
    reads W_b minus the eta-weighted gradients of tokens s <= t; the next chunk starts from W_b
    minus all of the chunk's weighted gradients. Every W_t is formed explicitly."""
    Q, K, V, eta = (torch.as_tensor(x, dtype=torch.float64) for x in (Q, K, V, eta))
    W = torch.as_tensor(W0, dtype=torch.float64).clone()
    O = torch.empty_like(Q)
    for c0 in range(0, Q.shape[0], C):
        grads = [eta[s] * _grad_inner_loss(W, K[s], V[s]) for s in range(c0, c0 + C)]
        for t in range(c0, c0 + C):
            Wt = W - sum(grads[: t - c0 + 1])
            O[t] = Q[t] @ Wt
        W = W - sum(grads)
    return O.numpy(), W.numpy()


# ----------------------------------------------------------------------------- dual form
@pytest.mark.parametrize("d,T", [(1, 5), (3, 7), (8, 16)])
def test_dual_C1_equals_per_token_sgd_autograd(d, T):
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.05, 0.4, T)
    W0 = _rand(d, d, scale=0.3)
    O, W = orc.dual_form_stream(Q, K, V, eta, W0, 1)
    O_ref, W_ref = _per_token_sgd(Q, K, V, eta, W0)
    np.testing.assert_allclose(O, O_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(W, W_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("d,T,C", [(2, 8, 2), (4, 12, 4), (8, 32, 8), (8, 32, 32), (5, 18, 3)])
def test_dual_equals_minibatch_gd_autograd(d, T, C):
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.05, 0.4, T)
    W0 = _rand(d, d, scale=0.3)
    O, W = orc.dual_form_stream(Q, K, V, eta, W0, C)
    O_ref, W_ref = _minibatch_gd_by_definition(Q, K, V, eta, W0, C)
    np.testing.assert_allclose(O, O_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(W, W_ref, rtol=1e-11, atol=1e-12)


def test_dual_scalar_eta_equals_constant_array():
    d, T, C = 4, 16, 4
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    W0 = _rand(d, d)
    a = orc.dual_form_stream(Q, K, V, 0.1, W0, C)
    b = orc.dual_form_stream(Q, K, V, np.full(T, 0.1), W0, C)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_dual_W0_zero_first_chunk_is_causal_linear_attention():
    """With W0 = 0 the first chunk's residuals are -V, so O = tril(Q K^T) diag(eta) V and
    W = K^T diag(eta) V: causal linear attention ("TTT with KV binding is in fact linear
    attention")."""
    d, C = 6, 8
    Q, K, V = _rand(C, d), _rand(C, d), _rand(C, d)
    eta = rng.uniform(0.1, 0.5, C)
    O, W = orc.dual_form_stream(Q, K, V, eta, None, C)
    O_la = np.array([sum(eta[s] * (Q[t] @ K[s]) * V[s] for s in range(t + 1)) for t in range(C)])
    W_la = sum(eta[s] * np.outer(K[s], V[s]) for s in range(C))
    np.testing.assert_allclose(O, O_la, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(W, W_la, rtol=1e-12, atol=1e-13)


def test_dual_chunked_differs_from_per_token():
    """The dual form equals the mini-batch update, not per-token SGD."""
    d, T = 4, 16
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    O1, W1 = orc.dual_form_stream(Q, K, V, 0.3, None, 1)
    O4, W4 = orc.dual_form_stream(Q, K, V, 0.3, None, 4)
    assert np.abs(O1 - O4).max() > 1e-3
    assert np.abs(W1 - W4).max() > 1e-3


def test_dual_state_carry_split_at_chunk_boundary():
    """Running T tokens equals running the first half, then the second from its final W."""
    d, T, C = 5, 24, 4
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.05, 0.3, T)
    W0 = _rand(d, d)
    O, W = orc.dual_form_stream(Q, K, V, eta, W0, C)
    h = 12
    Oa, Wa = orc.dual_form_stream(Q[:h], K[:h], V[:h], eta[:h], W0, C)
    Ob, Wb = orc.dual_form_stream(Q[h:], K[h:], V[h:], eta[h:], Wa, C)
    np.testing.assert_allclose(np.concatenate([Oa, Ob]), O, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Wb, W, rtol=1e-13, atol=1e-14)


def test_dual_batch_streams_independent_and_permutable():
    B, H, T, d, C = 2, 3, 8, 3, 4
    Q, K, V = _rand(B, H, T, d), _rand(B, H, T, d), _rand(B, H, T, d)
    eta = rng.uniform(0.05, 0.3, (B, H, T))
    W0 = _rand(B, H, d, d)
    O, W = orc.dual_form(Q, K, V, eta, W0, C)
    for b in range(B):
        for h in range(H):
            o, w = orc.dual_form_stream(Q[b, h], K[b, h], V[b, h], eta[b, h], W0[b, h], C)
            np.testing.assert_array_equal(O[b, h], o)
            np.testing.assert_array_equal(W[b, h], w)
    # subset selection returns exactly those streams, and threads do not change results
    Os, Ws = orc.dual_form(Q, K, V, eta, W0, C, streams=[(1, 2), (0, 1)], threads=2)
    np.testing.assert_array_equal(Os[0], O[1, 2])
    np.testing.assert_array_equal(Ws[1], W[0, 1])


def test_dual_rejects_ragged_T():
    with pytest.raises(ValueError):
        orc.dual_form_stream(_rand(10, 2), _rand(10, 2), _rand(10, 2), 0.1, None, 4)


# ----------------------------------------------------------------------------- associative mode
def test_assoc_one_token_closed_form_and_autograd_ascent():
    """o = q (S0 + k^T v) after one inner step ("TTT with KV binding is in fact linear
    attention"); the step is gradient ascent on <k S, v> with learning rate 1 (autograd)."""
    d = 5
    q, k, v = _rand(d), _rand(d), _rand(d)
    S0 = _rand(d, d)
    O, S = orc.assoc_recurrence_stream(q[None], k[None], v[None], 1.0, S0)
    np.testing.assert_allclose(O[0], q @ (S0 + np.outer(k, v)), rtol=1e-13)
    St = torch.tensor(S0, requires_grad=True)
    obj = (torch.tensor(k) @ St) @ torch.tensor(v)
    (g,) = torch.autograd.grad(obj, St)
    S1 = (St + 1.0 * g).detach().numpy()
    np.testing.assert_allclose(S, S1, rtol=1e-13)
    np.testing.assert_allclose(O[0], q @ S1, rtol=1e-13)


def test_assoc_each_step_is_ascent_with_token_eta():
    d, T = 3, 6
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.2, 1.0, T)
    S_prev = _rand(d, d)
    O, _ = orc.assoc_recurrence_stream(Q, K, V, eta, S_prev)
    for t in range(T):
        St = torch.tensor(S_prev, requires_grad=True)
        (g,) = torch.autograd.grad((torch.tensor(K[t]) @ St) @ torch.tensor(V[t]), St)
        S_prev = (St + eta[t] * g).detach().numpy()
        np.testing.assert_allclose(O[t], Q[t] @ S_prev, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T,C,L", [(24, 1, 24), (24, 4, 8), (24, 8, 24), (32, 8, 16), (30, 5, 10)])
def test_assoc_chunked_and_two_pass_equal_sequential(T, C, L):
    d = 4
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.1, 1.0, T)
    S0 = _rand(d, d)
    O, S = orc.assoc_recurrence_stream(Q, K, V, eta, S0)
    Oc, Sc = orc.assoc_chunked_stream(Q, K, V, eta, S0, C)
    Op, Sp = orc.assoc_two_pass_stream(Q, K, V, eta, S0, C, L)
    for a, b in ((Oc, O), (Sc, S), (Op, O), (Sp, S)):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_assoc_eta_folds_into_values():
    d, T = 4, 10
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.1, 1.0, T)
    O, S = orc.assoc_recurrence_stream(Q, K, V, eta, None)
    O2, S2 = orc.assoc_recurrence_stream(Q, K, eta[:, None] * V, 1.0, None)
    np.testing.assert_allclose(O, O2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, S2, rtol=1e-12, atol=1e-13)


def test_assoc_is_causal_linear_attention():
    d, T = 3, 9
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.1, 1.0, T)
    O, _ = orc.assoc_recurrence_stream(Q, K, V, eta, None)
    O_la = np.array([sum(eta[s] * (Q[t] @ K[s]) * V[s] for s in range(t + 1)) for t in range(T)])
    np.testing.assert_allclose(O, O_la, rtol=1e-12, atol=1e-13)


def test_assoc_all_streams_helper():
    B, H, T, d = 2, 2, 8, 3
    Q, K, V = _rand(B, H, T, d), _rand(B, H, T, d), _rand(B, H, T, d)
    eta = rng.uniform(0.1, 1.0, (B, H, T))
    O, S = orc.assoc_scan(Q, K, V, eta, None)
    Oc, Sc = orc.assoc_scan(Q, K, V, eta, None, form="chunked", C=4, threads=2)
    np.testing.assert_allclose(O, Oc, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, Sc, rtol=1e-12, atol=1e-13)
    o, s = orc.assoc_recurrence_stream(Q[1, 0], K[1, 0], V[1, 0], eta[1, 0], None)
    np.testing.assert_array_equal(O[1, 0], o)


# ----------------------------------------------------------------------------- In-Place TTT
def test_inplace_prefix_equals_block_strictly_causal_linear_attention():
    """O_i = Z_i W0 + eta sum_{j<i} (Z_i Z_j^T) Vhat_j: the prefix-sum form read as linear
    attention over earlier chunks only ("In-Place Test-Time Training", associative memory and
    associative-scan paragraphs)."""
    T, Dff, D, C, eta = 24, 7, 5, 6, 0.05
    Z, Vh, W0 = _rand(T, Dff), _rand(T, D), _rand(Dff, D)
    O, W = orc.inplace_chunks(Z, Vh, W0, eta, C)
    O_la = np.empty((T, D))
    for i0 in range(0, T, C):
        acc = Z[i0:i0 + C] @ W0
        for j0 in range(0, i0, C):
            acc = acc + eta * (Z[i0:i0 + C] @ Z[j0:j0 + C].T) @ Vh[j0:j0 + C]
        O_la[i0:i0 + C] = acc
    np.testing.assert_allclose(O, O_la, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(W, W0 + eta * Z.T @ Vh, rtol=1e-12, atol=1e-12)


def test_inplace_one_chunk_closed_form():
    T, Dff, D = 8, 6, 3
    Z, Vh, W0 = _rand(T, Dff), _rand(T, D), _rand(Dff, D)
    O, W = orc.inplace_chunks(Z, Vh, W0, 0.01, T)
    np.testing.assert_allclose(O, Z @ W0, rtol=1e-13)
    np.testing.assert_allclose(W, W0 + 0.01 * Z.T @ Vh, rtol=1e-13)


def test_inplace_delta_is_one_gradient_step_autograd():
    """The per-chunk delta is one step (learning rate eta) of descent on -<Z_i W, Vhat_i>."""
    T, Dff, D, eta = 4, 5, 3, 0.1
    Z, Vh, W0 = _rand(T, Dff), _rand(T, D), _rand(Dff, D)
    _, W = orc.inplace_chunks(Z, Vh, W0, eta, T)
    Wt = torch.tensor(W0, requires_grad=True)
    loss = -((torch.tensor(Z) @ Wt) * torch.tensor(Vh)).sum()
    (g,) = torch.autograd.grad(loss, Wt)
    np.testing.assert_allclose(W, (Wt - eta * g).detach().numpy(), rtol=1e-13)


def test_inplace_column_subset_is_exact():
    T, Dff, D, C = 12, 5, 9, 4
    Z, Vh, W0 = _rand(T, Dff), _rand(T, D), _rand(Dff, D)
    O, W = orc.inplace_chunks(Z, Vh, W0, 0.2, C)
    cols = [0, 4, 8]
    Os, Ws = orc.inplace_chunks(Z, Vh, W0, 0.2, C, cols=cols)
    np.testing.assert_array_equal(Os, O[:, cols])
    np.testing.assert_array_equal(Ws, W[:, cols])


# ----------------------------------------------------------------------------- hand-worked
def _golden():
    with open(GOLDEN) as f:
        g = json.load(f)
    g.pop("_about")
    return g


@pytest.mark.parametrize("name", sorted(_golden()))
def test_hand_worked_examples(name):
    ex = _golden()[name]
    if name.startswith("dual"):
        O, W = orc.dual_form_stream(ex["Q"], ex["K"], ex["V"], np.array(ex["eta"]), ex["W0"],
                                    ex["C"])
        np.testing.assert_allclose(W, ex["W"], rtol=0, atol=1e-15)
    elif name.startswith("assoc"):
        O, S = orc.assoc_recurrence_stream(ex["Q"], ex["K"], ex["V"], np.array(ex["eta"]),
                                           ex["S0"])
        np.testing.assert_allclose(S, ex["S"], rtol=0, atol=1e-15)
        Oc, _ = orc.assoc_chunked_stream(ex["Q"], ex["K"], ex["V"], np.array(ex["eta"]),
                                         ex["S0"], len(ex["Q"]))
        np.testing.assert_allclose(Oc, ex["O"], rtol=0, atol=1e-15)
    else:
        O, W = orc.inplace_chunks(ex["Z"], ex["Vhat"], ex["W0"], ex["eta"], ex["C"])
        np.testing.assert_allclose(W, ex["W"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(O, ex["O"], rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    """A plausible slip in the oracle (mask without the diagonal, eta on the target token, a
    sign flip) must fail the autograd pin. The slip is planted in a copy of the oracle's chunk
    step, on the CPU."""
    d, T, C = 4, 12, 4
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.05, 0.4, T)
    W0 = _rand(d, d, scale=0.3)
    O_ref, _ = _minibatch_gd_by_definition(Q, K, V, eta, W0, C)

    def variant(mask_k, eta_on_target, sign):
        W = W0.copy()
        O = np.empty((T, d))
        for c0 in range(0, T, C):
            q, k, v, e = Q[c0:c0 + C], K[c0:c0 + C], V[c0:c0 + C], eta[c0:c0 + C]
            G = k @ W - v
            A = np.tril(q @ k.T, mask_k) * (e[:, None] if eta_on_target else e[None, :])
            O[c0:c0 + C] = q @ W + sign * A @ G
            W = W - k.T @ (e[:, None] * G)
        return O

    assert np.allclose(variant(0, False, -1), O_ref, rtol=1e-11, atol=1e-12)
    for bad in ((-1, False, -1), (0, True, -1), (0, False, +1)):
        assert not np.allclose(variant(*bad), O_ref, rtol=1e-6, atol=1e-8)


# ----------------------------------------------------------------------------- associative backward
def _assoc_loss(Q, K, V, eta, S0, dO, G):
    """The scalar whose gradients the backward returns, from the forward definition only."""
    O, S = orc.assoc_recurrence_stream(Q, K, V, eta, S0)
    return float(np.sum(dO * O) + np.sum(G * S))


def _bwd_case(T, d, scalar_eta=False):
    Q, K, V, dO = _rand(T, d), _rand(T, d), _rand(T, d), _rand(T, d)
    eta = 0.3 if scalar_eta else rng.uniform(0.05, 0.9, T)
    S0, G = _rand(d, d, scale=0.5), _rand(d, d, scale=0.5)
    return Q, K, V, eta, S0, dO, G


def test_assoc_backward_matches_central_finite_differences():
    """Every gradient of the adjoint sweep against central differences of the forward
    definition (the loss is quadratic in each input, so the difference is exact up to
    rounding)."""
    Q, K, V, eta, S0, dO, G = _bwd_case(5, 3)
    dQ, dK, dV, deta, dS0 = orc.assoc_backward_stream(Q, K, V, eta, S0, dO, G)
    h = 1e-4
    args = [Q, K, V, eta, S0]
    for i, grad in enumerate((dQ, dK, dV, deta, dS0)):
        fd = np.empty_like(grad)
        for idx in np.ndindex(grad.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[i][idx] += h
            minus[i][idx] -= h
            fd[idx] = (_assoc_loss(*plus, dO, G) - _assoc_loss(*minus, dO, G)) / (2 * h)
        assert np.allclose(grad, fd, rtol=1e-7, atol=1e-8), i


@pytest.mark.parametrize("scalar_eta", [False, True])
def test_assoc_backward_matches_autograd(scalar_eta):
    """Against torch autograd of an independent restatement of the recurrence (float64)."""
    T, d = 24, 6
    Q, K, V, eta, S0, dO, G = _bwd_case(T, d, scalar_eta)
    dQ, dK, dV, deta, dS0 = orc.assoc_backward_stream(Q, K, V, eta, S0, dO, G)
    tq, tk, tv, ts0 = (torch.tensor(a, requires_grad=True) for a in (Q, K, V, S0))
    te = torch.tensor(np.full(T, eta) if scalar_eta else eta, requires_grad=True)
    S = ts0
    outs = []
    for t in range(T):
        S = S + te[t] * torch.outer(tk[t], tv[t])
        outs.append(tq[t] @ S)
    L = (torch.stack(outs) * torch.tensor(dO)).sum() + (S * torch.tensor(G)).sum()
    L.backward()
    for ours, ref in ((dQ, tq.grad), (dK, tk.grad), (dV, tv.grad), (deta, te.grad),
                      (dS0, ts0.grad)):
        assert np.allclose(ours, ref.numpy(), rtol=1e-10, atol=1e-11)


def test_assoc_backward_all_streams_helper_and_zero_inputs():
    """The batched helper equals the per-stream sweep; with dO = 0 and dS_out = 0 every gradient
    vanishes; with dO = 0 the state adjoint is dS_out throughout (dS0 = dS_out)."""
    B, H, T, d = 2, 2, 8, 3
    Q, K, V, dO = (_rand(B, H, T, d) for _ in range(4))
    eta = rng.uniform(0.1, 0.5, (B, H, T))
    G = _rand(B, H, d, d)
    out = orc.assoc_scan_bwd(Q, K, V, eta, None, dO, G)
    one = orc.assoc_backward_stream(Q[1, 0], K[1, 0], V[1, 0], eta[1, 0], None, dO[1, 0],
                                    G[1, 0])
    for a, b in zip(out, one):
        assert np.allclose(a[1, 0], b, rtol=0, atol=0)
    zero = orc.assoc_scan_bwd(Q, K, V, eta, None, np.zeros_like(dO), None)
    assert all(np.all(z == 0) for z in zero)
    only_g = orc.assoc_scan_bwd(Q, K, V, eta, None, np.zeros_like(dO), G)
    assert np.allclose(only_g[4], G) and np.all(only_g[0] == 0)


def test_assoc_backward_pins_catch_planted_mistakes():
    """Plausible slips in the adjoint (adding q_t^T dO_t after the token's gradients instead of
    before, a transposed state adjoint in dK, eta left out of dV) must fail the
    finite-difference pin. Planted in a copy of the reverse sweep, on the CPU."""
    Q, K, V, eta, S0, dO, G = _bwd_case(6, 3)
    ref = orc.assoc_backward_stream(Q, K, V, eta, S0, dO, G)

    def sweep(late_add, transpose_dk, drop_eta):
        A = G.copy()
        dK, dV = np.empty_like(K), np.empty_like(V)
        for t in range(len(Q) - 1, -1, -1):
            if not late_add:
                A += np.outer(Q[t], dO[t])
            kA = K[t] @ A
            dV[t] = (1.0 if drop_eta else eta[t]) * kA
            dK[t] = eta[t] * ((A.T if transpose_dk else A) @ V[t])
            if late_add:
                A += np.outer(Q[t], dO[t])
        return dK, dV

    good = sweep(False, False, False)
    assert np.allclose(good[0], ref[1]) and np.allclose(good[1], ref[2])
    for bad in ((True, False, False), (False, True, False), (False, False, True)):
        dK, dV = sweep(*bad)
        assert not (np.allclose(dK, ref[1], rtol=1e-6) and np.allclose(dV, ref[2], rtol=1e-6))


# ----------------------------------------------------------------------------- segment-affine scan
def test_dual_segment_maps_are_the_chunk_products_and_the_zero_start_run():
    """A is the product of the chunk matrices I - K_c^T diag(eta_c) K_c (latest on the left),
    formed here by a separate loop; B is the final state of the dual form started from W = 0;
    and for any start W the segment ends at A W + B."""
    T, d, C = 24, 5, 4
    K, V = _rand(T, d, scale=0.5), _rand(T, d)
    eta = rng.uniform(0.05, 0.6, T)
    A, B = orc.dual_segment_maps_stream(K, V, eta, C)
    P = np.eye(d)
    for c0 in range(0, T, C):
        k, e = K[c0:c0 + C], eta[c0:c0 + C]
        P = (np.eye(d) - k.T @ np.diag(e) @ k) @ P
    np.testing.assert_allclose(A, P, rtol=1e-12, atol=1e-13)
    Q = _rand(T, d)
    _, Wz = orc.dual_form_stream(Q, K, V, eta, None, C)
    np.testing.assert_allclose(B, Wz, rtol=1e-12, atol=1e-13)
    W0 = _rand(d, d)
    _, W = orc.dual_form_stream(Q, K, V, eta, W0, C)
    np.testing.assert_allclose(A @ W0 + B, W, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T,d,C,L", [(32, 4, 4, 8), (48, 6, 8, 16), (30, 3, 3, 6), (16, 4, 16, 16)])
def test_dual_segmented_equals_sequential(T, d, C, L):
    """Segment-affine composition equals the sequential chunk loop (any segment length that is
    a multiple of C), per-token and scalar rates, with and without W0."""
    Q, K, V = _rand(T, d), _rand(T, d, scale=0.5), _rand(T, d)
    for eta in (rng.uniform(0.05, 0.6, T), 0.3):
        for W0 in (None, _rand(d, d)):
            O, W = orc.dual_form_segmented_stream(Q, K, V, eta, W0, C, L)
            O_ref, W_ref = orc.dual_form_stream(Q, K, V, eta, W0, C)
            np.testing.assert_allclose(O, O_ref, rtol=1e-10, atol=1e-11)
            np.testing.assert_allclose(W, W_ref, rtol=1e-10, atol=1e-11)


def test_dual_segmented_rejects_bad_segment_lengths():
    Q = K = V = np.zeros((16, 2))
    for L in (0, 6, 32):   # not a positive multiple of C = 4 dividing T
        with pytest.raises(ValueError):
            orc.dual_form_segmented_stream(Q, K, V, 0.1, None, 4, L)


def test_dual_segment_maps_compose():
    """The map of two consecutive segments is the composition of their maps:
    (A2, B2) o (A1, B1) = (A2 A1, A2 B1 + B2), for any split at a chunk boundary."""
    T, d, C = 24, 4, 4
    K, V = _rand(T, d, scale=0.5), _rand(T, d)
    eta = rng.uniform(0.05, 0.6, T)
    A, B = orc.dual_segment_maps_stream(K, V, eta, C)
    for cut in (4, 12, 20):
        A1, B1 = orc.dual_segment_maps_stream(K[:cut], V[:cut], eta[:cut], C)
        A2, B2 = orc.dual_segment_maps_stream(K[cut:], V[cut:], eta[cut:], C)
        np.testing.assert_allclose(A2 @ A1, A, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(A2 @ B1 + B2, B, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- dual-form backward
def _dual_loss(Q, K, V, eta, W0, dO, G, C):
    """The scalar whose gradients the dual-form backward returns, from the forward only."""
    O, W = orc.dual_form_stream(Q, K, V, eta, W0, C)
    return float(np.sum(dO * O) + np.sum(G * W))


def _dual_bwd_case(T, d, scalar_eta=False, scale=0.6):
    Q, K, V, dO = (_rand(T, d, scale=scale) for _ in range(4))
    eta = 0.2 if scalar_eta else rng.uniform(0.05, 0.5, T)
    W0, G = _rand(d, d, scale=0.4), _rand(d, d, scale=0.5)
    return Q, K, V, eta, W0, dO, G


@pytest.mark.parametrize("T,d,C", [(6, 3, 3), (6, 2, 2), (4, 3, 4)])
def test_dual_backward_matches_central_finite_differences(T, d, C):
    """Every gradient of the chunk-wise adjoint against central differences of the forward
    (the loss is a polynomial in each input; h = 1e-5 leaves an O(h^2) truncation error)."""
    Q, K, V, eta, W0, dO, G = _dual_bwd_case(T, d)
    grads = orc.dual_backward_stream(Q, K, V, eta, W0, dO, G, C)
    h = 1e-5
    args = [Q, K, V, eta, W0]
    for i, grad in enumerate(grads):
        fd = np.empty_like(grad)
        for idx in np.ndindex(grad.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[i][idx] += h
            minus[i][idx] -= h
            fd[idx] = (_dual_loss(*plus, dO, G, C) - _dual_loss(*minus, dO, G, C)) / (2 * h)
        assert np.allclose(grad, fd, rtol=1e-6, atol=1e-8), i


def _inner_grad_graph(W, k, v):
    """Gradient of 1/2 ||k W - v||^2 at W by autograd, kept in the graph so that the outer
    loss can be differentiated through it."""
    loss = 0.5 * ((k @ W - v) ** 2).sum()
    (g,) = torch.autograd.grad(loss, W, create_graph=True)
    return g


@pytest.mark.parametrize("scalar_eta", [False, True])
@pytest.mark.parametrize("T,d,C", [(16, 4, 4), (12, 5, 3), (8, 3, 8)])
def test_dual_backward_matches_autograd_through_minibatch_steps(T, d, C, scalar_eta):
    """Against torch autograd of mini-batch TTT written by definition (every inner gradient
    taken by autograd at the chunk-start weight, every W_t formed explicitly), float64."""
    Q, K, V, eta, W0, dO, G = _dual_bwd_case(T, d, scalar_eta)
    grads = orc.dual_backward_stream(Q, K, V, eta, W0, dO, G, C)
    tq, tk, tv, tw = (torch.tensor(a, requires_grad=True) for a in (Q, K, V, W0))
    te = torch.tensor(np.full(T, eta) if scalar_eta else eta, requires_grad=True)
    W = tw
    outs = []
    for c0 in range(0, T, C):
        steps = [te[s] * _inner_grad_graph(W, tk[s], tv[s]) for s in range(c0, c0 + C)]
        for t in range(c0, c0 + C):
            outs.append(tq[t] @ (W - sum(steps[: t - c0 + 1])))
        W = W - sum(steps)
    L = (torch.stack(outs) * torch.tensor(dO)).sum() + (W * torch.tensor(G)).sum()
    L.backward()
    for ours, ref in zip(grads, (tq.grad, tk.grad, tv.grad, te.grad, tw.grad)):
        assert np.allclose(ours, ref.numpy(), rtol=1e-9, atol=1e-11)


def test_dual_backward_zero_keys_closed_form_and_helper():
    """With K = 0 the state never moves: dQ = dO W0^T, dV = 0, deta = 0 and
    dW0 = dW_out + Q^T dO. The batched helper equals the per-stream sweep, and zero output
    gradients give zero everywhere."""
    T, d, C = 12, 4, 4
    Q, _, V, eta, W0, dO, G = _dual_bwd_case(T, d)
    dQ, dK, dV, deta, dW0 = orc.dual_backward_stream(Q, np.zeros((T, d)), V, eta, W0, dO, G, C)
    assert np.allclose(dQ, dO @ W0.T, rtol=1e-13, atol=1e-13)
    assert np.all(dV == 0) and np.allclose(deta, 0, atol=1e-15)
    assert np.allclose(dW0, G + Q.T @ dO, rtol=1e-13, atol=1e-13)
    B, H = 2, 2
    Qb, Kb, Vb, dOb = (_rand(B, H, T, d, scale=0.5) for _ in range(4))
    eb = rng.uniform(0.1, 0.5, (B, H, T))
    Gb = _rand(B, H, d, d)
    out = orc.dual_form_bwd(Qb, Kb, Vb, eb, None, dOb, Gb, C)
    one = orc.dual_backward_stream(Qb[1, 0], Kb[1, 0], Vb[1, 0], eb[1, 0], None, dOb[1, 0],
                                   Gb[1, 0], C)
    for a, b in zip(out, one):
        assert np.array_equal(a[1, 0], b)
    zero = orc.dual_form_bwd(Qb, Kb, Vb, eb, None, np.zeros_like(dOb), None, C)
    assert all(np.all(z == 0) for z in zero)


def test_dual_backward_pins_catch_planted_mistakes():
    """Plausible slips in the chunk adjoint (the causal mask without its diagonal, the -A^T dO
    term left out of dG, the state after the chunk used in place of the chunk-start state) must
    fail the finite-difference pin. Planted in a copy of the reverse sweep, on the CPU."""
    T, d, C = 6, 3, 3
    Q, K, V, eta, W0, dO, G = _dual_bwd_case(T, d)
    fd_dq = np.empty((T, d))
    for idx in np.ndindex(T, d):
        plus, minus = Q.copy(), Q.copy()
        plus[idx] += 1e-5
        minus[idx] -= 1e-5
        fd_dq[idx] = (_dual_loss(plus, K, V, eta, W0, dO, G, C)
                      - _dual_loss(minus, K, V, eta, W0, dO, G, C)) / 2e-5
    fd_w0 = np.empty((d, d))
    for idx in np.ndindex(d, d):
        plus, minus = W0.copy(), W0.copy()
        plus[idx] += 1e-5
        minus[idx] -= 1e-5
        fd_w0[idx] = (_dual_loss(Q, K, V, eta, plus, dO, G, C)
                      - _dual_loss(Q, K, V, eta, minus, dO, G, C)) / 2e-5

    def sweep(strict_mask, drop_at_do, end_state):
        W, starts = W0.copy(), []
        for c0 in range(0, T, C):
            starts.append(W.copy())
            k, v, e = K[c0:c0 + C], V[c0:c0 + C], eta[c0:c0 + C]
            W = W - k.T @ (e[:, None] * (k @ W - v))
        starts.append(W)
        mask = np.tril(np.ones((C, C)), -1 if strict_mask else 0)
        X, dq_all = G.copy(), np.empty((T, d))
        for ci in range(T // C - 1, -1, -1):
            sl = slice(ci * C, ci * C + C)
            q, k, v, e, do = Q[sl], K[sl], V[sl], eta[sl], dO[sl]
            W = starts[ci + 1] if end_state else starts[ci]
            Gc = k @ W - v
            A = (q @ k.T) * mask * e[None, :]
            dG = -e[:, None] * (k @ X) - (0 if drop_at_do else A.T @ do)
            dQK = -(do @ Gc.T) * mask * e[None, :]
            dq_all[sl] = do @ W.T + dQK @ k
            X = X + q.T @ do + k.T @ dG
        return dq_all, X

    good = sweep(False, False, False)
    assert np.allclose(good[0], fd_dq, rtol=1e-6, atol=1e-8)
    assert np.allclose(good[1], fd_w0, rtol=1e-6, atol=1e-8)
    for bad in ((True, False, False), (False, True, False), (False, False, True)):
        dq, dw0 = sweep(*bad)
        assert not (np.allclose(dq, fd_dq, rtol=1e-4) and np.allclose(dw0, fd_w0, rtol=1e-4))


def test_backwards_are_linear_in_the_incoming_gradients():
    """Both backwards are linear maps of (dO, dState): the gradients for a combination of two
    incoming gradients are the same combination of their gradients (catches a term that squares
    or drops an incoming gradient)."""
    T, d, C = 8, 3, 4
    Q, K, V = _rand(T, d), _rand(T, d, scale=0.5), _rand(T, d)
    eta = rng.uniform(0.05, 0.5, T)
    W0 = _rand(d, d, scale=0.3)
    dO1, dO2 = _rand(T, d), _rand(T, d)
    G1, G2 = _rand(d, d), _rand(d, d)
    a, b = 0.7, -1.3
    for fn in (lambda o, g: orc.dual_backward_stream(Q, K, V, eta, W0, o, g, C),
               lambda o, g: orc.assoc_backward_stream(Q, K, V, eta, W0, o, g)):
        g1, g2 = fn(dO1, G1), fn(dO2, G2)
        gc = fn(a * dO1 + b * dO2, a * G1 + b * G2)
        for x1, x2, xc in zip(g1, g2, gc):
            np.testing.assert_allclose(xc, a * x1 + b * x2, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------- momentum
def test_momentum_beta_zero_is_the_plain_recurrence():
    T, d = 20, 5
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.1, 0.6, T)
    S0 = _rand(d, d)
    O, S, M = orc.assoc_momentum_stream(Q, K, V, eta, 0.0, S0, None)
    Or, Sr = orc.assoc_recurrence_stream(Q, K, V, eta, S0)
    assert np.allclose(O, Or, rtol=1e-12, atol=1e-12) and np.allclose(S, Sr, rtol=1e-12)
    assert np.allclose(M, eta[-1] * np.outer(K[-1], V[-1]), rtol=1e-12)


@pytest.mark.parametrize("beta", [0.5, 0.9, 0.99])
def test_momentum_closed_weighted_sum(beta):
    """Unrolled, the momentum form is a linear-attention sum with weights
    (1 - beta^(t-s+1)) / (1 - beta) on token s's update, plus the initial momentum's
    contribution beta (1 - beta^t) / (1 - beta) M0 after t tokens (t counted from 1)."""
    T, d = 17, 4
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.1, 0.6, T)
    S0, M0 = _rand(d, d), _rand(d, d)
    O, S, M = orc.assoc_momentum_stream(Q, K, V, eta, beta, S0, M0)
    for t in range(T):
        n = t + 1
        St = S0 + beta * (1 - beta ** n) / (1 - beta) * M0
        for s_ in range(t + 1):
            St = St + (1 - beta ** (t - s_ + 1)) / (1 - beta) * eta[s_] * np.outer(K[s_], V[s_])
        assert np.allclose(O[t], Q[t] @ St, rtol=1e-10, atol=1e-12)
    Mt = beta ** T * M0 + sum(beta ** (T - 1 - s_) * eta[s_] * np.outer(K[s_], V[s_])
                              for s_ in range(T))
    assert np.allclose(M, Mt, rtol=1e-10, atol=1e-12)


def test_momentum_beta_one_closed_form():
    """beta = 1: the momentum is the running sum of the updates and the state its running sum,
    so token s's update enters S_t with weight t - s + 1 and M0 with weight t (t counted from 1)."""
    T, d = 13, 3
    Q, K, V = _rand(T, d), _rand(T, d), _rand(T, d)
    eta = rng.uniform(0.1, 0.6, T)
    S0, M0 = _rand(d, d), _rand(d, d)
    O, S, M = orc.assoc_momentum_stream(Q, K, V, eta, 1.0, S0, M0)
    for t in range(T):
        St = S0 + (t + 1) * M0
        for s_ in range(t + 1):
            St = St + (t - s_ + 1) * eta[s_] * np.outer(K[s_], V[s_])
        assert np.allclose(O[t], Q[t] @ St, rtol=1e-10, atol=1e-12)
    assert np.allclose(M, M0 + sum(eta[s_] * np.outer(K[s_], V[s_]) for s_ in range(T)),
                       rtol=1e-10, atol=1e-12)
    assert np.allclose(S, St, rtol=1e-10, atol=1e-12)


def test_momentum_two_tokens_by_hand():
    """d = 1: q = (1, 2), k = (1, 1), v = (3, 5), eta = (0.5, 1), beta = 0.5, S0 = M0 = 0.
    M1 = 1.5, S1 = 1.5, o1 = 1.5; M2 = 0.75 + 5 = 5.75, S2 = 7.25, o2 = 14.5."""
    O, S, M = orc.assoc_momentum_stream([[1.0], [2.0]], [[1.0], [1.0]], [[3.0], [5.0]],
                                        [0.5, 1.0], 0.5, None, None)
    assert np.allclose(O[:, 0], [1.5, 14.5]) and np.isclose(S[0, 0], 7.25)
    assert np.isclose(M[0, 0], 5.75)


def test_momentum_all_streams_helper():
    B, H, T, d = 2, 3, 6, 3
    Q, K, V = _rand(B, H, T, d), _rand(B, H, T, d), _rand(B, H, T, d)
    O, S, M = orc.assoc_momentum(Q, K, V, 0.25, 0.8, None, None)
    o, s_, m = orc.assoc_momentum_stream(Q[1, 2], K[1, 2], V[1, 2], 0.25, 0.8, None, None)
    assert np.array_equal(O[1, 2], o) and np.array_equal(S[1, 2], s_)
    assert np.array_equal(M[1, 2], m)


# ----------------------------------------------------------------------------- LM-aligned target
def test_lm_target_brute_force():
    """Against the definition written as plain loops on a tiny case."""
    T, Dm, D, k = 7, 3, 2, 4
    X, Wc, Wp = _rand(T, Dm), _rand(k, Dm), _rand(Dm, D)
    got = orc.lm_target(X, Wc, Wp)
    ref = np.zeros((T, D))
    for t in range(T):
        for n in range(D):
            acc = 0.0
            for j in range(Dm):
                for i in range(k):
                    tt = t + 1 - i
                    if 0 <= tt < T:
                        acc += Wc[i, j] * X[tt, j] * Wp[j, n]
            ref[t, n] = acc
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_lm_target_single_taps_and_causality():
    """Tap 1 alone reads the current token (Vhat = X Wp); tap 0 alone reads the next one (and
    zero at the last token); Vhat_t changes with X_(t+1) but not with X_(t+2)."""
    T, Dm, D = 9, 4, 3
    X, Wp = _rand(T, Dm), _rand(Dm, D)
    cur = np.zeros((4, Dm))
    cur[1] = 1.0
    assert np.allclose(orc.lm_target(X, cur, Wp), X @ Wp, rtol=1e-12)
    nxt = np.zeros((4, Dm))
    nxt[0] = 1.0
    ref = np.vstack([X[1:] @ Wp, np.zeros((1, D))])
    assert np.allclose(orc.lm_target(X, nxt, Wp), ref, rtol=1e-12, atol=1e-14)
    Wc = _rand(4, Dm)
    base = orc.lm_target(X, Wc, Wp)
    X2 = X.copy()
    X2[5] += 1.0
    d = orc.lm_target(X2, Wc, Wp) - base
    assert np.abs(d[4]).max() > 1e-6           # token 4 sees token 5 (the next one)
    assert np.abs(d[:4]).max() == 0.0           # earlier tokens do not see two ahead
