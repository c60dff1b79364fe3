"""The stage form of the dual-form backward, in fp64 on the CPU, against the oracle's chunk-wise
adjoint ("RNN의 기억을 작은 모델로 바꾼다면: Test-Time Training 읽기", section "gradient를
효율적인 layer로 만드는 작업": the mini-batch updates are differentiated with the layer).

The GPU kernel for d = 64 does not evaluate the per-chunk adjoint statement by statement. Per
128-token stage it uses the stage-start state W_s and the state gradient X_e after the stage's
last chunk, with -E = -diag(eta) G as the operand of its tensor-core products:

    dQ = dO W_s^T + P1 K                     P1[t][s] = [s <= t] (dO (-E)^T)[t][s]
    dK = P1^T Q + (-E) X_e^T + dG W_s^T + P2 K + P2^T K
                                             P2[a][b] = [chunk(b) < chunk(a)] (dG (-E)^T)[a][b]
    dV = -dG,  deta_s = (-E_s . R_s) / eta_s  (= -G_s . R_s; G itself where eta_s is tiny)

with R = A'^T dO + K X and dG = -diag(eta) R per chunk (A' = tril(Q K^T) of the chunk). This file
evaluates those identities step by step in numpy and checks them against the oracle, so that a
mistake in the stage algebra (a mask off by one chunk, a missing transposed term, a sign) fails
here, on the CPU, independently of the kernel.
"""
import numpy as np
import pytest

from oracle import ttt_oracle as orc

C = 16
R_STAGE = 128


def stage_form_backward(Q, K, V, eta, W0, dO, dW_out, tiny=1e-20, mistake=None):
    """One stream, fp64: forward chunk states, then the stage form of the backward. `mistake`
    plants one error in the stage algebra (for the test that the comparison notices it)."""
    T, d = Q.shape
    eta = np.broadcast_to(np.asarray(eta, dtype=np.float64), (T,))
    # forward: chunk-start states, residuals
    W = W0.copy()
    G = np.zeros((T, d))
    W_stage = []
    for c0 in range(0, T, C):
        if c0 % R_STAGE == 0:
            W_stage.append(W.copy())
        sl = slice(c0, c0 + C)
        G[sl] = K[sl] @ W - V[sl]
        W = W - K[sl].T @ (eta[sl, None] * G[sl])
    NE = -eta[:, None] * G
    dQ, dK, dV = np.zeros((T, d)), np.zeros((T, d)), np.zeros((T, d))
    deta = np.zeros(T)
    X = dW_out.copy()
    n_stage = (T + R_STAGE - 1) // R_STAGE
    for j in reversed(range(n_stage)):
        s0, s1 = j * R_STAGE, min((j + 1) * R_STAGE, T)
        st = slice(s0, s1)
        n = s1 - s0
        X_e = X.copy()
        dG = np.zeros((n, d))
        # the chain, chunks from the last
        for c0 in reversed(range(s0, s1, C)):
            sl = slice(c0, c0 + C)
            Ap = np.tril(Q[sl] @ K[sl].T)           # A'[t][s], s <= t
            R = Ap.T @ dO[sl] + K[sl] @ X
            g = -eta[sl, None] * R
            dG[c0 - s0:c0 - s0 + C] = g
            e = eta[sl]
            big = np.abs(e) >= tiny
            de = np.where(big, np.sum(NE[sl] * R, axis=1) / np.where(big, e, 1.0),
                          -np.sum(G[sl] * R, axis=1))
            deta[sl] = de
            X = X + Q[sl].T @ dO[sl] + K[sl].T @ g
        # the stage products
        tok = np.arange(n)
        S1 = dO[st] @ NE[st].T
        if mistake == "p1_strict":
            P1 = np.where(tok[None, :] < tok[:, None], S1, 0.0)
        else:
            P1 = np.where(tok[None, :] <= tok[:, None], S1, 0.0)
        S2 = dG @ NE[st].T
        if mistake == "p2_inclusive":
            P2 = np.where((tok[None, :] // C) <= (tok[:, None] // C), S2, 0.0)
        else:
            P2 = np.where((tok[None, :] // C) < (tok[:, None] // C), S2, 0.0)
        Ws = W_stage[j]
        dQ[st] = dO[st] @ Ws.T + P1 @ K[st]
        dK[st] = P1.T @ Q[st] + dG @ Ws.T + P2 @ K[st]
        if mistake != "no_p2t":
            dK[st] += P2.T @ K[st]
        if mistake != "no_xe":
            dK[st] += NE[st] @ X_e.T
        dV[st] = -dG
    return dQ, dK, dV, deta, X


def _inputs(T, d, seed, eta_kind="random"):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((T, d)) / np.sqrt(d)
    K = rng.standard_normal((T, d))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((T, d))
    V /= np.linalg.norm(V, axis=1, keepdims=True)
    if eta_kind == "random":
        eta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    elif eta_kind == "with_zeros":
        eta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
        eta[3] = 0.0
        eta[130:150] = 0.0
        eta[17] = 1e-25
    else:
        eta = np.zeros(T)
    W0 = 0.02 * rng.standard_normal((d, d))
    dO = rng.standard_normal((T, d))
    dW = 0.05 * rng.standard_normal((d, d))
    return Q, K, V, eta, W0, dO, dW


@pytest.mark.parametrize("T,d,kind", [(16, 8, "random"), (272, 8, "random"), (384, 16, "random"),
                                      (272, 8, "with_zeros"), (160, 8, "zeros")])
def test_stage_form_equals_chunk_adjoint(T, d, kind):
    Q, K, V, eta, W0, dO, dW = _inputs(T, d, seed=T + d, eta_kind=kind)
    got = stage_form_backward(Q, K, V, eta, W0, dO, dW)
    ref = orc.dual_backward_stream(Q, K, V, eta, W0, dO, dW, C)
    for name, g, r in zip(("dQ", "dK", "dV", "deta", "dW0"), got, ref):
        scale = max(1.0, float(np.abs(r).max()))
        assert np.abs(g - r).max() <= 1e-10 * scale, name


@pytest.mark.parametrize("mistake", ["p1_strict", "p2_inclusive", "no_p2t", "no_xe"])
def test_planted_stage_algebra_mistakes_are_caught(mistake):
    """P1 without its diagonal, P2 with the diagonal chunk, the transposed P2 term dropped, the
    X_e term dropped: each breaks the agreement with the chunk-wise adjoint."""
    Q, K, V, eta, W0, dO, dW = _inputs(272, 8, seed=3)
    ref = orc.dual_backward_stream(Q, K, V, eta, W0, dO, dW, C)
    got = stage_form_backward(Q, K, V, eta, W0, dO, dW, mistake=mistake)
    errs = [np.abs(g - r).max() / max(1.0, float(np.abs(r).max())) for g, r in zip(got, ref)]
    assert max(errs) > 1e-4, (mistake, errs)
