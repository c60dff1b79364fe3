"""Seeded synthetic inputs for the three fast-weight workloads.

This module holds the input recipe only: the distributions, the per-token L2 normalisation of
keys/values, the per-token learning-rate squashing and the rounding to the storage dtype. It holds
none of the update-and-read arithmetic. Both the CUDA path and the fp64 oracle consume the tensors
returned here (the oracle widens them to float64), so the two sides always see identical values.

Generation uses a torch generator on the requested device (``cpu`` or ``cuda``), seeded per
workload; draws happen in a fixed order so a (workload, seed, device) triple always yields the same
tensors. Values are drawn in fp32, normalised in fp32 and only then rounded (round-to-nearest-even)
to bf16 where the workload stores bf16, so the rounded keys are not exactly unit-norm.

Workloads mirror the shapes the pages discuss: TTT-Linear layers of the 125M and 1.3B models
("Learning to (Learn at Test Time)" reading, section on long-context results), the weight-norm-free
linear-attention form ("TTT with KV binding is in fact linear attention", associativity paragraph)
and the In-Place TTT W_down update on a 4B-class MLP ("In-Place Test-Time Training", chunk update
paragraph).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: kind is 'dual', 'assoc' or 'inplace'."""

    name: str
    kind: str
    seed: int
    B: int = 1
    H: int = 1
    T: int = 0
    d: int = 0
    C: int = 0
    dtype: str = "bf16"
    # dual / assoc recipe switches
    qkv: str = "normal"          # 'normal' = N(0,1); 'normal_1_over_d' = N(0, 1/d)
    normalise: tuple = ()        # subset of ('Q','K','V') that are L2-normalised per token
    eta: str = "sigmoid_over_d"  # 'sigmoid_over_d' | 'sigmoid' | 'const'
    eta_const: float = 0.0
    w0: str = "normal_0.02"      # 'normal_0.02' | 'zero'
    # in-place recipe
    Dff: int = 0
    D: int = 0
    # LM-aligned target (in-place with its target formed from embeddings)
    Dm: int = 0
    k: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.T if not self.kind.startswith("inplace") else self.T


# The five workloads of the forward path use seeds 1000 + i; the backward of the associative
# mode and its momentum form, on the associative workload's shape, use 1005 and 1007.
MOMENTUM_BETA = 0.9   # momentum coefficient of the momentum workload
WORKLOADS = {
    "dual_f32_B1H2T256_d32C16": Workload(
        "dual_f32_B1H2T256_d32C16", "dual", 1000, B=1, H=2, T=256, d=32, C=16, dtype="f32",
        qkv="normal_1_over_d", normalise=(), eta="const", eta_const=0.1, w0="zero"),
    "dual_bf16_B8H12T2048_d64C16": Workload(
        "dual_bf16_B8H12T2048_d64C16", "dual", 1001, B=8, H=12, T=2048, d=64, C=16,
        normalise=("K", "V")),
    "dual_bf16_B2H32T32768_d64C16": Workload(
        "dual_bf16_B2H32T32768_d64C16", "dual", 1002, B=2, H=32, T=32768, d=64, C=16,
        normalise=("K", "V")),
    "assoc_bf16_B4H16T65536_d128C64": Workload(
        "assoc_bf16_B4H16T65536_d128C64", "assoc", 1003, B=4, H=16, T=65536, d=128, C=64,
        normalise=("Q", "K"), eta="sigmoid", w0="zero"),
    "inplace_bf16_T32768_Dff9728_D2560_C1024": Workload(
        "inplace_bf16_T32768_Dff9728_D2560_C1024", "inplace", 1004, T=32768, C=1024,
        Dff=9728, D=2560, eta="const", eta_const=1e-3),
    "assoc_momentum_bf16_B4H16T65536_d128C64": Workload(
        "assoc_momentum_bf16_B4H16T65536_d128C64", "assoc_momentum", 1007, B=4, H=16, T=65536,
        d=128, C=64, normalise=("Q", "K"), eta="sigmoid", w0="zero"),
    "inplace_lm_bf16_T32768_Dff9728_D2560_Dm2560_C1024": Workload(
        "inplace_lm_bf16_T32768_Dff9728_D2560_Dm2560_C1024", "inplace_lm", 1008, T=32768,
        C=1024, Dff=9728, D=2560, Dm=2560, k=4, eta="const", eta_const=1e-3),
    "dual_bf16_B1H4T262144_d64C16": Workload(
        "dual_bf16_B1H4T262144_d64C16", "dual", 1010, B=1, H=4, T=262144, d=64, C=16,
        normalise=("K", "V")),
    "dual_seg_bf16_B1H4T262144_d64C16": Workload(
        "dual_seg_bf16_B1H4T262144_d64C16", "dual_seg", 1010, B=1, H=4, T=262144, d=64, C=16,
        normalise=("K", "V")),
    "dual_bwd_bf16_B1H4T262144_d64C16": Workload(
        "dual_bwd_bf16_B1H4T262144_d64C16", "dual_bwd", 1011, B=1, H=4, T=262144, d=64, C=16,
        normalise=("K", "V")),
    "dual_seg_bwd_bf16_B1H4T262144_d64C16": Workload(
        "dual_seg_bwd_bf16_B1H4T262144_d64C16", "dual_seg_bwd", 1011, B=1, H=4, T=262144,
        d=64, C=16, normalise=("K", "V")),
    "dual_bwd_bf16_B8H12T2048_d64C16": Workload(
        "dual_bwd_bf16_B8H12T2048_d64C16", "dual_bwd", 1006, B=8, H=12, T=2048, d=64, C=16,
        normalise=("K", "V")),
    "assoc_bwd_bf16_B4H16T65536_d128C64": Workload(
        "assoc_bwd_bf16_B4H16T65536_d128C64", "assoc_bwd", 1005, B=4, H=16, T=65536, d=128,
        C=64, normalise=("Q", "K"), eta="sigmoid", w0="zero"),
    # the associative mode at head dim 64 and a 16-token chunk (evaluated on 64-token tiles)
    "assoc_bf16_B4H16T65536_d64C16": Workload(
        "assoc_bf16_B4H16T65536_d64C16", "assoc", 1012, B=4, H=16, T=65536, d=64, C=16,
        normalise=("Q", "K"), eta="sigmoid", w0="zero"),
}
WORKLOAD_ORDER = list(WORKLOADS)


def _torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _l2_normalise(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def dual_or_assoc_inputs(B: int, H: int, T: int, d: int, *, seed: int, device="cpu",
                         dtype: str = "bf16", qkv: str = "normal", normalise=(),
                         eta: str = "sigmoid_over_d", eta_const: float = 0.0,
                         w0: str = "normal_0.02") -> dict:
    """Q, K, V [B,H,T,d] in ``dtype``; eta [B,H,T] fp32 (or None with ``eta_scalar``);
    W0 [B,H,d,d] fp32. Draw order: Q, K, V, z (for eta), W0."""
    g = _gen(seed, device)
    std = 1.0 if qkv == "normal" else (1.0 / d) ** 0.5
    shape = (B, H, T, d)
    out = {}
    for name in ("Q", "K", "V"):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std
        if name in normalise:
            x = _l2_normalise(x)
        out[name] = x.to(_torch_dtype(dtype)).contiguous()
    if eta == "const":
        out["eta"] = None
        out["eta_scalar"] = float(eta_const)
    else:
        z = torch.randn((B, H, T), generator=g, device=device, dtype=torch.float32)
        e = torch.sigmoid(z)
        if eta == "sigmoid_over_d":
            e = e / d
        out["eta"] = e.contiguous()
        out["eta_scalar"] = 0.0
    if w0 == "zero":
        out["W0"] = torch.zeros((B, H, d, d), device=device, dtype=torch.float32)
    else:
        out["W0"] = (torch.randn((B, H, d, d), generator=g, device=device,
                                 dtype=torch.float32) * 0.02).contiguous()
    return out


def inplace_inputs(T: int, Dff: int, D: int, *, seed: int, device="cpu",
                   eta: float = 1e-3, row_block: int = 4096) -> dict:
    """Z [T,Dff] bf16 = silu(A) * Bm with A, Bm ~ N(0,1); Vhat [T,D] bf16 ~ N(0, 0.02^2);
    W0 [Dff,D] bf16 ~ N(0, 0.02^2). Draw order: A, Bm (row block by row block), Vhat, W0."""
    g = _gen(seed, device)
    Z = torch.empty((T, Dff), device=device, dtype=torch.bfloat16)
    for r0 in range(0, T, row_block):
        r1 = min(T, r0 + row_block)
        a = torch.randn((r1 - r0, Dff), generator=g, device=device, dtype=torch.float32)
        b = torch.randn((r1 - r0, Dff), generator=g, device=device, dtype=torch.float32)
        Z[r0:r1] = (torch.nn.functional.silu(a) * b).to(torch.bfloat16)
    Vhat = (torch.randn((T, D), generator=g, device=device, dtype=torch.float32) * 0.02
            ).to(torch.bfloat16)
    W0 = (torch.randn((Dff, D), generator=g, device=device, dtype=torch.float32) * 0.02
          ).to(torch.bfloat16)
    return {"Z": Z, "Vhat": Vhat, "W0": W0, "eta": float(eta)}


def assoc_bwd_inputs(B: int, H: int, T: int, d: int, *, seed: int, device="cpu",
                     **recipe) -> dict:
    """The associative inputs of ``dual_or_assoc_inputs`` (S0 = 0) plus the incoming gradients:
    dO [B,H,T,d] bf16 ~ N(0,1) and dS_out [B,H,d,d] fp32 ~ N(0, 0.05^2), drawn in that order
    from a generator seeded with seed + 1."""
    out = dual_or_assoc_inputs(B, H, T, d, seed=seed, device=device, **recipe)
    g = _gen(seed + 1, device)
    out["dO"] = torch.randn((B, H, T, d), generator=g, device=device,
                            dtype=torch.float32).to(torch.bfloat16).contiguous()
    out["dS_out"] = (torch.randn((B, H, d, d), generator=g, device=device,
                                 dtype=torch.float32) * 0.05).contiguous()
    return out


def dual_bwd_inputs(B: int, H: int, T: int, d: int, *, seed: int, device="cpu",
                    **recipe) -> dict:
    """The dual-form inputs of ``dual_or_assoc_inputs`` plus the incoming gradients:
    dO [B,H,T,d] bf16 ~ N(0,1) and dW_out [B,H,d,d] fp32 ~ N(0, 0.05^2), drawn in that order
    from a generator seeded with seed + 1."""
    out = dual_or_assoc_inputs(B, H, T, d, seed=seed, device=device, **recipe)
    g = _gen(seed + 1, device)
    out["dO"] = torch.randn((B, H, T, d), generator=g, device=device,
                            dtype=torch.float32).to(torch.bfloat16).contiguous()
    out["dW_out"] = (torch.randn((B, H, d, d), generator=g, device=device,
                                 dtype=torch.float32) * 0.05).contiguous()
    return out


def inplace_lm_inputs(T: int, Dff: int, D: int, Dm: int, k: int, *, seed: int, device="cpu",
                      eta: float = 1e-3) -> dict:
    """The In-Place inputs of ``inplace_inputs`` (its Vhat is not used) plus the embeddings and
    target weights: X [T, Dm] bf16 ~ N(0,1); Wc [k, Dm] fp32 ~ N(0, 1/k) (so the convolved
    embeddings have unit variance); Wp [Dm, D] bf16 ~ N(0, 0.02^2 / Dm) (so Vhat has the
    N(0, 0.02^2) scale of the plain recipe), drawn in that order from a generator seeded
    seed + 1."""
    out = inplace_inputs(T, Dff, D, seed=seed, device=device, eta=eta)
    del out["Vhat"]
    g = _gen(seed + 1, device)
    out["X"] = torch.randn((T, Dm), generator=g, device=device,
                           dtype=torch.float32).to(torch.bfloat16)
    out["Wc"] = (torch.randn((k, Dm), generator=g, device=device, dtype=torch.float32)
                 * (1.0 / k) ** 0.5).contiguous()
    out["Wp"] = (torch.randn((Dm, D), generator=g, device=device, dtype=torch.float32)
                 * (0.02 / Dm ** 0.5)).to(torch.bfloat16)
    return out


def make_inputs(w: Workload, device="cpu", *, seed: Optional[int] = None, **overrides) -> dict:
    """Inputs of a named workload (optionally with shape overrides for reduced cases)."""
    if overrides:
        w = dataclasses.replace(w, **overrides)
    s = w.seed if seed is None else seed
    if w.kind in ("dual", "dual_seg", "assoc", "assoc_momentum"):
        return dual_or_assoc_inputs(w.B, w.H, w.T, w.d, seed=s, device=device, dtype=w.dtype,
                                    qkv=w.qkv, normalise=w.normalise, eta=w.eta,
                                    eta_const=w.eta_const, w0=w.w0)
    if w.kind == "assoc_bwd":
        return assoc_bwd_inputs(w.B, w.H, w.T, w.d, seed=s, device=device, dtype=w.dtype,
                                qkv=w.qkv, normalise=w.normalise, eta=w.eta,
                                eta_const=w.eta_const, w0=w.w0)
    if w.kind in ("dual_bwd", "dual_seg_bwd"):
        return dual_bwd_inputs(w.B, w.H, w.T, w.d, seed=s, device=device, dtype=w.dtype,
                               qkv=w.qkv, normalise=w.normalise, eta=w.eta,
                               eta_const=w.eta_const, w0=w.w0)
    if w.kind == "inplace":
        return inplace_inputs(w.T, w.Dff, w.D, seed=s, device=device, eta=w.eta_const)
    if w.kind == "inplace_lm":
        return inplace_lm_inputs(w.T, w.Dff, w.D, w.Dm, w.k, seed=s, device=device,
                                 eta=w.eta_const)
    raise ValueError(w.kind)
