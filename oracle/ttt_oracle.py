"""fp64 CPU oracle for the chunked fast-weight update-and-read. TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module. The CUDA library never calls it, and nothing here calls the CUDA library: the two
share no code. Inputs are the exact values the GPU receives (bf16 tensors widened to float64,
the same fp32 learning rates); every result is float64.

Sources, cited by page title and the passage on it:

  [TTT-read]  "RNN의 기억을 작은 모델로 바꾼다면: Test-Time Training 읽기" (ariser.io), a reading
              of "Learning to (Learn at Test Time)". Section "읽는 동안 문제를 하나 더 푼다":
              the per-token rule W_t = W_(t-1) - eta * grad l(W_(t-1); x_t), output read from the
              *updated* model. Section "gradient를 효율적인 layer로 만드는 작업": mini-batch TTT and
              its dual form, which equals the mini-batch update (not per-token SGD).
              Section "원문의 긴 문맥 결과를 읽는 범위": state reset per sequence, batch items kept
              apart.
  [KVB]       "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다" (aitrends.kr): one inner
              step with a linear bias-free last layer gives o = q(S0 + k^T v); without weight
              normalisation the state update is associative (parallel prefix scan); per-token
              learning rates fold into the values; gradient ascent in the inner loop.
  [IPT]       "In-Place 테스트 시점 학습: LLM을 위한 원활한 동적 적응 프레임워크" (aitrends.kr):
              W_down of the gated MLP is the fast weight, refreshed once per chunk (C = 512..1024)
              with one gradient step; the updated weight serves the *next* chunk; per-chunk deltas
              combine by a prefix sum (associative scan), equal to the sequential update.

Readings where the pages leave a step open (each also listed in the design notes):
  * inner loss 1/2 ||k W - v||^2 with row vectors and W laid out [d_in][d_out], so the gradient
    of token s at W is k_s^T (k_s W - v_s);
  * the intra-chunk causal mask includes the diagonal (token t sees its own gradient, as the
    per-token rule reads the updated model);
  * a per-token learning rate scales the *source* token's gradient (or value);
  * the associative mode adds eta_t k_t^T v_t (ascent on <k S, v>) and reads o_t = q_t S_t after
    the update of token t;
  * the In-Place chunk i reads W0 plus the deltas of chunks strictly before it, and the delta is
    +eta Z_i^T Vhat_i.

Pins (tests/test_oracle_pins.py): per-token SGD from autograd gradients at C=1; mini-batch
gradient descent from autograd gradients at any C; the causal-linear-attention closed form at
W0 = 0; o = q(S0 + k^T v) for one token; the sequential recurrence vs. the chunked and two-pass
forms; eta folded into V; the In-Place block-causal linear-attention form and its one-chunk closed
form; autograd ascent steps for the associative and In-Place deltas; hand-worked golden examples;
the associative backward against central finite differences of the forward definition and
against autograd of an independent torch restatement; the dual-form backward against central
finite differences and against autograd through mini-batch gradient steps that autograd itself
takes; the momentum recurrence against the plain one at beta = 0, against its closed
weighted-sum form and against hand-worked tokens; the segment maps of the dual form against
the product of the chunk matrices and the zero-start dual form, and the segmented evaluation
against the sequential chunk loop. Every function below has at least one pin.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Sequence

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _eta_stream(eta, T: int) -> np.ndarray:
    if np.ndim(eta) == 0:
        return np.full(T, float(eta))
    e = _f64(eta)
    assert e.shape == (T,)
    return e


# --------------------------------------------------------------------------------------------
# TTT-Linear, mini-batch dual form  [TTT-read, "gradient를 효율적인 layer로 만드는 작업"]
# --------------------------------------------------------------------------------------------
def dual_form_stream(Q, K, V, eta, W0, C: int):
    """One (batch, head) stream. Q, K, V: [T, d]; eta: [T] or scalar; W0: [d, d] or None (zeros).

    For each chunk of C tokens, with W the state at the chunk's start:
        G   = K_c W - V_c                      (residuals; token s's gradient is k_s^T g_s)
        O_c = Q_c W - (tril(Q_c K_c^T) * eta_s) G
              i.e. token t reads W minus the eta-weighted gradients of tokens s <= t of its chunk
        W   = W - K_c^T diag(eta_c) G          (one mini-batch step at the chunk-start W)
    Returns (O [T, d], W_final [d, d]).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    T, d = Q.shape
    if C <= 0 or T % C:
        raise ValueError("T must be a positive multiple of C")
    e_all = _eta_stream(eta, T)
    W = np.zeros((d, d)) if W0 is None else _f64(W0).copy()
    O = np.empty((T, d))
    for c0 in range(0, T, C):
        q, k, v, e = Q[c0:c0 + C], K[c0:c0 + C], V[c0:c0 + C], e_all[c0:c0 + C]
        G = k @ W - v
        A = np.tril(q @ k.T) * e[None, :]
        O[c0:c0 + C] = q @ W - A @ G
        W = W - k.T @ (e[:, None] * G)
    return O, W


def _streams(fn, arrays, B: int, H: int, threads: int, streams: Optional[Sequence] = None):
    idx = list(streams) if streams is not None else [(b, h) for b in range(B) for h in range(H)]
    if threads <= 1:
        return idx, [fn(b, h) for (b, h) in idx]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return idx, list(ex.map(lambda bh: fn(*bh), idx))


def dual_form(Q, K, V, eta, W0, C: int, *, threads: int = 1, streams=None):
    """All (b, h) streams of [B, H, T, d] inputs; eta [B, H, T] or scalar; W0 [B, H, d, d] or
    None. Streams are independent [TTT-read, "원문의 긴 문맥 결과를 읽는 범위"].
    ``streams`` selects a subset of (b, h) pairs; the result then holds only those, in order:
    (O [n, T, d], W [n, d, d]). Without it the result is (O [B,H,T,d], W [B,H,d,d])."""
    B, H, T, d = np.shape(Q)

    def one(b, h):
        e = eta if np.ndim(eta) == 0 else np.asarray(eta)[b, h]
        w0 = None if W0 is None else np.asarray(W0)[b, h]
        return dual_form_stream(np.asarray(Q)[b, h], np.asarray(K)[b, h], np.asarray(V)[b, h],
                                e, w0, C)

    idx, res = _streams(one, None, B, H, threads, streams)
    O = np.stack([r[0] for r in res])
    W = np.stack([r[1] for r in res])
    if streams is None:
        O = O.reshape(B, H, T, d)
        W = W.reshape(B, H, d, d)
    return O, W


def dual_segment_maps_stream(K, V, eta, C: int):
    """The chunk updates of one segment of tokens composed into one affine map
    W_end = A W_start + B [KVB, associativity paragraph: without weight normalisation the
    update is associative; applied here to the dual form's affine chunk update
    W' = (I - K^T diag(eta) K) W + K^T diag(eta) V]. Propagates the pair (A, B) from (I, 0)
    through the segment's chunks in order. Returns (A [d, d], B [d, d])."""
    K, V = _f64(K), _f64(V)
    T, d = K.shape
    if C <= 0 or T % C:
        raise ValueError("T must be a positive multiple of C")
    e_all = _eta_stream(eta, T)
    A, B = np.eye(d), np.zeros((d, d))
    for c0 in range(0, T, C):
        k, v, e = K[c0:c0 + C], V[c0:c0 + C], e_all[c0:c0 + C]
        A = A - k.T @ (e[:, None] * (k @ A))
        B = B - k.T @ (e[:, None] * (k @ B - v))
    return A, B


def dual_form_segmented_stream(Q, K, V, eta, W0, C: int, L: int):
    """Sequence-parallel evaluation of ``dual_form_stream``: the sequence is cut into segments of
    L tokens (L a multiple of C); each segment's map (A_s, B_s) comes from
    ``dual_segment_maps_stream``; the segment start states follow by folding the maps in order,
    W_start(s+1) = A_s W_start(s) + B_s; every segment then runs the dual form from its start
    state. Returns (O [T, d], W_final [d, d]); equal to ``dual_form_stream`` up to rounding."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    T, d = Q.shape
    if L <= 0 or L % C or T % L:
        raise ValueError("L must be a positive multiple of C that divides T")
    e_all = _eta_stream(eta, T)
    W = np.zeros((d, d)) if W0 is None else _f64(W0).copy()
    starts = []
    for s0 in range(0, T, L):
        starts.append(W.copy())
        A, B = dual_segment_maps_stream(K[s0:s0 + L], V[s0:s0 + L], e_all[s0:s0 + L], C)
        W = A @ W + B
    O = np.empty((T, d))
    for i, s0 in enumerate(range(0, T, L)):
        O[s0:s0 + L], W_end = dual_form_stream(Q[s0:s0 + L], K[s0:s0 + L], V[s0:s0 + L],
                                               e_all[s0:s0 + L], starts[i], C)
    return O, W_end


def dual_backward_stream(Q, K, V, eta, W0, dO, dW_out, C: int):
    """Gradients of  L = sum_t <dO_t, o_t> + <dW_out, W_T>  through the dual form of
    ``dual_form_stream`` (the backward pass that outer-loop training of the layer needs
    [TTT-read, "gradient를 효율적인 layer로 만드는 작업"]: the inner updates are differentiated
    like any other layer).

    A forward sweep recomputes the chunk-start states W_c. A reverse sweep carries X, the
    gradient of L with respect to the state after the chunk (dW_out after the last one), and
    differentiates the chunk's three statements in reverse order:
        W' = W - K^T diag(eta) G :  dW += X,  dG = -diag(eta) K X,
                                    dk_s = -eta_s g_s X^T,  deta_s = -k_s X g_s^T
        O  = Q W - A G, A = tril(Q K^T) diag(eta) :
                                    dW += Q^T dO,  dG += -A^T dO,
                                    dA = -tril(dO G^T)  (entries s > t of A are zero),
                                    d(QK^T) = dA diag(eta) -> dQ += d(QK^T) K, dK += d(QK^T)^T Q,
                                    deta_s += sum_t dA[t, s] (Q K^T)[t, s]
        G  = K W - V :              dW += K^T dG,  dK += dG W^T,  dV = -dG
    and the total dW is X for the chunk before. After chunk 0, X is dW0.
    Returns (dQ, dK, dV [T, d], deta [T] (per token; their sum when eta is a scalar),
    dW0 [d, d])."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    T, d = Q.shape
    if C <= 0 or T % C:
        raise ValueError("T must be a positive multiple of C")
    e_all = _eta_stream(eta, T)
    W = np.zeros((d, d)) if W0 is None else _f64(W0).copy()
    starts = []
    for c0 in range(0, T, C):                             # forward sweep: chunk-start states
        starts.append(W.copy())
        k, v, e = K[c0:c0 + C], V[c0:c0 + C], e_all[c0:c0 + C]
        W = W - k.T @ (e[:, None] * (k @ W - v))
    X = np.zeros((d, d)) if dW_out is None else _f64(dW_out).copy()
    dQ, dK, dV, deta = np.empty((T, d)), np.empty((T, d)), np.empty((T, d)), np.empty(T)
    mask = np.tril(np.ones((C, C)))
    for ci in range(T // C - 1, -1, -1):                  # reverse sweep
        c0 = ci * C
        sl = slice(c0, c0 + C)
        q, k, v, e, do = Q[sl], K[sl], V[sl], e_all[sl], dO[sl]
        W = starts[ci]
        G = k @ W - v
        QK = q @ k.T
        A = QK * mask * e[None, :]
        # W' = W - K^T diag(eta) G
        kX = k @ X
        dG = -e[:, None] * kX
        dk = -e[:, None] * (G @ X.T)
        de = -np.sum(kX * G, axis=1)
        # O = Q W - A G
        dW = X + q.T @ do
        dG = dG - A.T @ do
        dA = -(do @ G.T) * mask
        dQK = dA * e[None, :]
        dq = do @ W.T + dQK @ k
        dk = dk + dQK.T @ q
        de = de + np.sum(dA * QK, axis=0)
        # G = K W - V
        dW = dW + k.T @ dG
        dk = dk + dG @ W.T
        dQ[sl], dK[sl], dV[sl], deta[sl] = dq, dk, -dG, de
        X = dW
    return dQ, dK, dV, deta, X


def dual_form_bwd(Q, K, V, eta, W0, dO, dW_out, C: int, *, threads: int = 1, streams=None):
    """All streams of [B, H, T, d] inputs (eta [B, H, T] or scalar; W0 / dW_out [B, H, d, d] or
    None). Returns (dQ, dK, dV, deta, dW0); deta is per token even for a scalar eta."""
    B, H, T, d = np.shape(Q)

    def one(b, h):
        e = eta if np.ndim(eta) == 0 else np.asarray(eta)[b, h]
        w0 = None if W0 is None else np.asarray(W0)[b, h]
        g = None if dW_out is None else np.asarray(dW_out)[b, h]
        return dual_backward_stream(np.asarray(Q)[b, h], np.asarray(K)[b, h],
                                    np.asarray(V)[b, h], e, w0, np.asarray(dO)[b, h], g, C)

    idx, res = _streams(one, None, B, H, threads, streams)
    out = [np.stack([r[i] for r in res]) for i in range(5)]
    if streams is None:
        shapes = [(B, H, T, d)] * 3 + [(B, H, T), (B, H, d, d)]
        out = [o.reshape(sh) for o, sh in zip(out, shapes)]
    return tuple(out)


# --------------------------------------------------------------------------------------------
# Associative (weight-norm-free, gradient-ascent) linear-attention mode  [KVB]
# --------------------------------------------------------------------------------------------
def assoc_recurrence_stream(Q, K, V, eta, S0):
    """Sequential definition, one token at a time: S_t = S_(t-1) + eta_t k_t^T v_t, o_t = q_t S_t.
    The chunk size does not enter. Returns (O [T, d], S_final [d, d])."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    T, d = Q.shape
    e = _eta_stream(eta, T)
    S = np.zeros((d, d)) if S0 is None else _f64(S0).copy()
    O = np.empty((T, d))
    for t in range(T):
        S += e[t] * np.outer(K[t], V[t])
        O[t] = Q[t] @ S
    return O, S


def assoc_chunked_stream(Q, K, V, eta, S0, C: int):
    """Chunk form of the same recurrence: per chunk, O_c = Q_c S + (tril(Q_c K_c^T) * eta_s) V_c,
    then S += K_c^T diag(eta_c) V_c. Equal to the sequential form by associativity [KVB]."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    T, d = Q.shape
    if C <= 0 or T % C:
        raise ValueError("T must be a positive multiple of C")
    e_all = _eta_stream(eta, T)
    S = np.zeros((d, d)) if S0 is None else _f64(S0).copy()
    O = np.empty((T, d))
    for c0 in range(0, T, C):
        q, k, v, e = Q[c0:c0 + C], K[c0:c0 + C], V[c0:c0 + C], e_all[c0:c0 + C]
        O[c0:c0 + C] = q @ S + (np.tril(q @ k.T) * e[None, :]) @ v
        S = S + k.T @ (e[:, None] * v)
    return O, S


def assoc_two_pass_stream(Q, K, V, eta, S0, C: int, L: int):
    """Two-pass prefix-scan form over superchunks of L tokens (L a multiple of C):
    pass 1 sums each superchunk's state increment; an exclusive prefix sum (plus S0) gives each
    superchunk's starting state; pass 2 runs the chunk form inside each superchunk from it
    [KVB, associativity paragraph; IPT, associative-scan paragraph]."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    T, d = Q.shape
    if L <= 0 or L % C or T % L:
        raise ValueError("T must be a multiple of L, and L a multiple of C")
    e_all = _eta_stream(eta, T)
    starts = list(range(0, T, L))
    deltas = [K[s:s + L].T @ (e_all[s:s + L, None] * V[s:s + L]) for s in starts]      # pass 1
    S = np.zeros((d, d)) if S0 is None else _f64(S0).copy()
    S_start = []
    for dS in deltas:                                                                  # scan
        S_start.append(S.copy())
        S = S + dS
    O = np.empty((T, d))
    for s, Ss in zip(starts, S_start):                                                 # pass 2
        O[s:s + L], _ = assoc_chunked_stream(Q[s:s + L], K[s:s + L], V[s:s + L],
                                             e_all[s:s + L], Ss, C)
    return O, S


def assoc_scan(Q, K, V, eta, S0, *, threads: int = 1, streams=None, form: str = "sequential",
               C: int = 64):
    """All streams; ``form`` picks 'sequential' (the definition) or 'chunked' (pinned equal)."""
    B, H, T, d = np.shape(Q)

    def one(b, h):
        e = eta if np.ndim(eta) == 0 else np.asarray(eta)[b, h]
        s0 = None if S0 is None else np.asarray(S0)[b, h]
        q, k, v = np.asarray(Q)[b, h], np.asarray(K)[b, h], np.asarray(V)[b, h]
        if form == "sequential":
            return assoc_recurrence_stream(q, k, v, e, s0)
        return assoc_chunked_stream(q, k, v, e, s0, C)

    idx, res = _streams(one, None, B, H, threads, streams)
    O = np.stack([r[0] for r in res])
    S = np.stack([r[1] for r in res])
    if streams is None:
        O = O.reshape(B, H, T, d)
        S = S.reshape(B, H, d, d)
    return O, S


def assoc_momentum_stream(Q, K, V, eta, beta: float, S0, M0):
    """Associative mode with a momentum inner loop [KVB, momentum paragraph: with momentum SGD
    the layer is still a weighted sum of linear-attention terms], one token at a time:
        M_t = beta M_(t-1) + eta_t k_t^T v_t,   S_t = S_(t-1) + M_t,   o_t = q_t S_t
    (the ascent gradient of <k S, v> is k^T v; the rate scales each token's gradient before it
    enters the momentum; M_0 = M0, zeros by default). Returns (O [T, d], S_T, M_T)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    T, d = Q.shape
    e = _eta_stream(eta, T)
    S = np.zeros((d, d)) if S0 is None else _f64(S0).copy()
    M = np.zeros((d, d)) if M0 is None else _f64(M0).copy()
    O = np.empty((T, d))
    for t in range(T):
        M = beta * M + e[t] * np.outer(K[t], V[t])
        S = S + M
        O[t] = Q[t] @ S
    return O, S, M


def assoc_momentum(Q, K, V, eta, beta: float, S0, M0, *, threads: int = 1, streams=None):
    """All streams of [B, H, T, d] inputs; S0 / M0 [B, H, d, d] or None. Returns (O, S_T, M_T)."""
    B, H, T, d = np.shape(Q)

    def one(b, h):
        e = eta if np.ndim(eta) == 0 else np.asarray(eta)[b, h]
        s0 = None if S0 is None else np.asarray(S0)[b, h]
        m0 = None if M0 is None else np.asarray(M0)[b, h]
        return assoc_momentum_stream(np.asarray(Q)[b, h], np.asarray(K)[b, h],
                                     np.asarray(V)[b, h], e, beta, s0, m0)

    idx, res = _streams(one, None, B, H, threads, streams)
    out = [np.stack([r[i] for r in res]) for i in range(3)]
    if streams is None:
        out = [out[0].reshape(B, H, T, d), out[1].reshape(B, H, d, d),
               out[2].reshape(B, H, d, d)]
    return tuple(out)


def assoc_backward_stream(Q, K, V, eta, S0, dO, dS_out):
    """Gradients of  L = sum_t <dO_t, o_t> + <dS_out, S_T>  through the associative recurrence
    S_t = S_(t-1) + eta_t k_t^T v_t, o_t = q_t S_t (the backward pass that outer-loop training
    of the layer needs).

    Written as the adjoint of the recurrence, one token at a time. A forward sweep recomputes
    S_t and gives dq_t = dO_t S_t^T. A reverse sweep carries the state adjoint A (the gradient
    of L with respect to S_t): A starts at dS_out; token t first adds q_t^T dO_t (o_t reads S_t),
    then dv_t = eta_t k_t A, dk_t = eta_t v_t A^T and deta_t = k_t A v_t^T; A passes to S_(t-1)
    unchanged because S_t = S_(t-1) + ... . After token 0, A is dS0.
    Returns (dQ, dK, dV [T, d], deta [T] (per-token rates; their sum when eta is a scalar),
    dS0 [d, d])."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    T, d = Q.shape
    e = _eta_stream(eta, T)
    S = np.zeros((d, d)) if S0 is None else _f64(S0).copy()
    dQ = np.empty((T, d))
    for t in range(T):                                    # forward sweep
        S += e[t] * np.outer(K[t], V[t])
        dQ[t] = dO[t] @ S.T
    A = np.zeros((d, d)) if dS_out is None else _f64(dS_out).copy()
    dK, dV, deta = np.empty((T, d)), np.empty((T, d)), np.empty(T)
    for t in range(T - 1, -1, -1):                        # reverse sweep
        A += np.outer(Q[t], dO[t])
        kA = K[t] @ A
        dV[t] = e[t] * kA
        dK[t] = e[t] * (A @ V[t])
        deta[t] = kA @ V[t]
    return dQ, dK, dV, deta, A


def assoc_scan_bwd(Q, K, V, eta, S0, dO, dS_out, *, threads: int = 1, streams=None):
    """All streams of [B, H, T, d] inputs (eta [B, H, T] or scalar, S0 / dS_out [B, H, d, d] or
    None). Returns (dQ, dK, dV, deta, dS0); deta is per token even for a scalar eta."""
    B, H, T, d = np.shape(Q)

    def one(b, h):
        e = eta if np.ndim(eta) == 0 else np.asarray(eta)[b, h]
        s0 = None if S0 is None else np.asarray(S0)[b, h]
        g = None if dS_out is None else np.asarray(dS_out)[b, h]
        return assoc_backward_stream(np.asarray(Q)[b, h], np.asarray(K)[b, h],
                                     np.asarray(V)[b, h], e, s0, np.asarray(dO)[b, h], g)

    idx, res = _streams(one, None, B, H, threads, streams)
    out = [np.stack([r[i] for r in res]) for i in range(5)]
    if streams is None:
        shapes = [(B, H, T, d)] * 3 + [(B, H, T), (B, H, d, d)]
        out = [o.reshape(sh) for o, sh in zip(out, shapes)]
    return tuple(out)


# --------------------------------------------------------------------------------------------
# In-Place TTT W_down chunk update  [IPT]
# --------------------------------------------------------------------------------------------
def inplace_chunks(Z, Vhat, W0, eta: float, C: int, cols=None):
    """Z [T, Dff]; Vhat [T, D]; W0 [Dff, D]. Sequentially over chunks i of C tokens:
        O_i = Z_i W          (W = W0 plus the deltas of the chunks before i)
        W   = W + eta Z_i^T Vhat_i
    Returns (O [T, D'], W_final [Dff, D']) where D' = len(cols) when ``cols`` selects output
    columns (each column of O and W depends only on the same column of Vhat and W0, so a column
    subset is exact, not an approximation)."""
    T, Dff = np.shape(Z)
    if C <= 0 or T % C:
        raise ValueError("T must be a positive multiple of C")
    Vh = np.asarray(Vhat)
    W = np.asarray(W0)
    if cols is not None:
        Vh = Vh[:, cols]
        W = W[:, cols]
    W = _f64(W).copy()
    O = np.empty((T, W.shape[1]))
    for c0 in range(0, T, C):
        z = _f64(np.asarray(Z)[c0:c0 + C])
        O[c0:c0 + C] = z @ W
        W = W + eta * (z.T @ _f64(Vh[c0:c0 + C]))
    return O, W


# --------------------------------------------------------------------------------------------
# LM-aligned target for the In-Place update  [IPT, LM-aligned objective paragraph]
# --------------------------------------------------------------------------------------------
def lm_target(X, Wc, Wp):
    """Vhat = conv(X) Wp: a depthwise 1D convolution over tokens that reaches one token ahead,
    then a bias-free projection [IPT: the target is made from the token embeddings by a 1D
    convolution and a projection and carries the next token's information].
    X [T, Dm]; Wc [k, Dm] (tap i multiplies token t + 1 - i: the next token, the current one and
    k - 2 before it; tokens outside [0, T) count as zero); Wp [Dm, D]. Returns Vhat [T, D]."""
    X, Wc, Wp = _f64(X), _f64(Wc), _f64(Wp)
    T, Dm = X.shape
    U = np.zeros((T, Dm))
    for i in range(Wc.shape[0]):
        shift = 1 - i                      # U[t] += Wc[i] * X[t + shift]
        lo, hi = max(0, -shift), min(T, T - shift)
        U[lo:hi] += Wc[i][None, :] * X[lo + shift:hi + shift]
    return U @ Wp
