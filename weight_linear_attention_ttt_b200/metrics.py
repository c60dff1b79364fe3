"""Algorithmic work of each operation: the flops and bytes the method itself must compute and
move, used for roofline fractions. Workspace, superchunk-state and re-read traffic is NOT
counted: it is overhead a kernel has to beat.

Dual form, per token and head: K_c W, Q_c W, K_c^T G (2 d^2 flops each) plus the intra-chunk
scores Q_c K_c^T and their product with G (2 C d each): 6 d^2 + 4 C d flops. Bytes: Q, K, V in
and O out (d elements each) plus one fp32 learning rate, and per stream the fp32 state in and out.

Associative mode, per token and head: Q S and K^T V (2 d^2 each) plus the causal C x C terms
(4 C d, counted dense): 4 d^2 + 4 C d flops; bytes as the dual form.

Dual-form backward, per token and head: 14 d^2 + 10 C d flops (see ``algorithmic``); bytes: Q, K,
V, dO in, dQ, dK, dV out, eta in, deta out, and per stream three fp32 d x d states.

In-Place, per token: the read Z_i W and the update Z_i^T Vhat_i, 2 Dff D flops each; bytes: Z,
Vhat, W0 (bf16), O (bf16) and the final fp32 W once each.
"""
from __future__ import annotations

import dataclasses

from .inputs import Workload


def algorithmic(w: Workload) -> dict:
    """{'flops': F, 'bytes': B, 'tokens': N} for one call of the workload."""
    if w.kind == "assoc_momentum":
        # the momentum recurrence reads and writes what the plain one does, plus the momentum
        # state (in and out); flops: the chunk steps of both states, about twice the plain
        # recurrence's
        a = algorithmic(dataclasses.replace(w, kind="assoc"))
        return {"flops": 2 * a["flops"], "bytes": a["bytes"] + w.B * w.H * 2 * w.d * w.d * 4,
                "tokens": a["tokens"]}
    if w.kind == "dual_seg":
        # the same operation as the dual form; the two extra passes are overhead
        return algorithmic(dataclasses.replace(w, kind="dual"))
    if w.kind in ("dual", "assoc"):
        e = 4 if w.dtype == "f32" else 2
        th = w.B * w.H * w.T
        per_tok = (6 if w.kind == "dual" else 4) * w.d * w.d + 4 * w.C * w.d
        eta_bytes = 4 if w.eta != "const" else 0
        state_bytes = 2 * w.d * w.d * 4
        return {"flops": th * per_tok,
                "bytes": th * (4 * w.d * e + eta_bytes) + w.B * w.H * state_bytes,
                "tokens": w.B * w.T}
    if w.kind == "assoc_bwd":
        # three passes of the forward recurrence (dQ, and dV / dK through the state gradient);
        # bytes: Q, K, V, dO in and dQ, dK, dV out (bf16), eta in and deta out (fp32), per
        # stream dS_out in and dS0 out (the initial state is zero)
        th = w.B * w.H * w.T
        return {"flops": 3 * th * (4 * w.d * w.d + 4 * w.C * w.d),
                "bytes": th * (7 * w.d * 2 + 8) + w.B * w.H * 2 * w.d * w.d * 4,
                "tokens": w.B * w.T}
    if w.kind == "dual_seg_bwd":
        return algorithmic(dataclasses.replace(w, kind="dual_bwd"))
    if w.kind == "dual_bwd":
        # the chunk adjoint's products: K W, K X, dO W^T, dG W^T, diag(eta) G X^T, Q^T dO and
        # K^T dG (2 d^2 each) plus the C x C terms Q K^T, dO G^T, A^T dO, dS K, dS^T Q (2 C d
        # each); recomputing the chunk-start states is overhead and not counted. Bytes: Q, K,
        # V, dO in and dQ, dK, dV out (bf16), eta in and deta out (fp32), per stream W0 and
        # dW_out in and dW0 out (fp32)
        th = w.B * w.H * w.T
        return {"flops": th * (14 * w.d * w.d + 10 * w.C * w.d),
                "bytes": th * (7 * w.d * 2 + 8) + w.B * w.H * 3 * w.d * w.d * 4,
                "tokens": w.B * w.T}
    if w.kind == "inplace_lm":
        # the In-Place update plus the target: convolution (2 k Dm flops per token) and
        # projection (2 Dm D per token); bytes: the update's with Vhat replaced by X, Wc, Wp
        a = algorithmic(dataclasses.replace(w, kind="inplace"))
        T, Dm, D = w.T, w.Dm, w.D
        return {"flops": a["flops"] + T * (2 * w.k * Dm + 2 * Dm * D),
                "bytes": a["bytes"] - T * D * 2 + T * Dm * 2 + w.k * Dm * 4 + Dm * D * 2,
                "tokens": T}
    if w.kind == "inplace":
        T, F, D = w.T, w.Dff, w.D
        return {"flops": 4 * F * D * T,
                "bytes": T * F * 2 + T * D * 2 + F * D * 2 + T * D * 2 + F * D * 4,
                "tokens": T}
    raise ValueError(w.kind)


def roofline_seconds(w: Workload, hbm_gbs: float, tensor_tflops: float) -> tuple:
    """(seconds, bound) = the slower of flops at the tensor peak and bytes at HBM bandwidth."""
    a = algorithmic(w)
    t_flops = a["flops"] / (tensor_tflops * 1e12)
    t_bytes = a["bytes"] / (hbm_gbs * 1e9)
    return (t_bytes, "hbm") if t_bytes >= t_flops else (t_flops, "tensor")
