"""Context parallelism: the sequence of every stream is split over ranks (associative mode and
dual form).

Without weight normalisation the associative state update composes by addition ("KV 바인딩 기반
테스트 시간 학습은 사실상 선형 어텐션이다", associativity paragraph), so a sequence split into
slices can be evaluated slice-parallel with one exchange step ("In-Place 테스트 시점 학습",
associative-scan paragraph: per-chunk deltas combined by a prefix sum equal the sequential
update):

  1. every rank computes its slice's state increment dS_r = sum_t eta_t k_t^T v_t
     (`ttt_assoc_state_fwd`);
  2. the increments are all-gathered over the process group (NCCL on GPUs): B*H*d*d fp32 per
     rank, a few MB;
  3. rank r starts from S0 + sum_{r' < r} dS_r' (`ttt_state_prefix_sum`) and runs the
     associative scan on its slice (`ttt_assoc_scan_fwd`);
  4. the state after the whole sequence, S0 + sum_r dS_r, is formed on every rank.

The compute steps are the library's kernels; torch.distributed carries only the all-gather. The
callables can be replaced (the CPU tests pass fp64 oracle functions) to test the orchestration
without a GPU.
"""
from __future__ import annotations

from typing import Callable, Optional


def assoc_scan_fwd_cp(Q, K, V, eta=None, S0=None, *, C: int, eta_scalar: float = 0.0,
                      group=None, state_fn: Optional[Callable] = None,
                      scan_fn: Optional[Callable] = None,
                      prefix_fn: Optional[Callable] = None):
    """This rank's slice (tokens [t_r, t_{r+1}) of every stream, contiguous [B,H,T_r,d]) ->
    (O_slice, S_final). S0 [B,H,d,d] (or None) is the same on every rank; S_final is the state
    after the whole sequence, identical on every rank."""
    import torch
    import torch.distributed as dist

    from . import ttt_assoc_scan_fwd, ttt_assoc_state_fwd, ttt_state_prefix_sum

    state_fn = state_fn or (lambda K_, V_, e_: ttt_assoc_state_fwd(
        K_, V_, e_, C=C, eta_scalar=eta_scalar))
    scan_fn = scan_fn or (lambda Q_, K_, V_, e_, s_: ttt_assoc_scan_fwd(
        Q_, K_, V_, e_, s_, C=C, eta_scalar=eta_scalar))
    prefix_fn = prefix_fn or (lambda s0, inc, upto: ttt_state_prefix_sum(s0, inc, upto))

    dS = state_fn(K, V, eta)
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    gathered = torch.empty((world,) + tuple(dS.shape), dtype=dS.dtype, device=dS.device)
    if world > 1:
        dist.all_gather(list(gathered.unbind(0)), dS.contiguous(), group=group)
    else:
        gathered[0].copy_(dS)
    start = prefix_fn(S0, gathered, rank)
    O, _ = scan_fn(Q, K, V, eta, start)
    S_final = prefix_fn(S0, gathered, world)
    return O, S_final


def dual_form_fwd_cp(Q, K, V, eta=None, W0=None, *, C: int, eta_scalar: float = 0.0,
                     group=None, maps_fn: Optional[Callable] = None,
                     scan_fn: Optional[Callable] = None, fold_fn: Optional[Callable] = None):
    """Dual form over a sequence split across ranks. The chunk update is affine in the state
    once weight normalisation is gone, so a rank's slice maps its start state by
    W_end = A_r W_start + B_r:

      1. every rank computes its slice's maps (A_r, B_r) (`ttt_linear_dual_slice_maps`);
      2. the maps are all-gathered (2 B*H*d*d fp32 per rank);
      3. rank r folds the maps of ranks r' < r onto W0 (`ttt_dual_state_fold`) and runs the dual
         form on its slice from there (`ttt_linear_dual_fwd`);
      4. the state after the whole sequence is the fold of all the maps, on every rank.

    This rank's slice is tokens [t_r, t_{r+1}) of every stream, contiguous [B,H,T_r,d] (T_r a
    multiple of C). Returns (O_slice, W_final). The callables can be replaced (the CPU tests
    pass fp64 oracle functions)."""
    import torch
    import torch.distributed as dist

    from . import ttt_dual_state_fold, ttt_linear_dual_fwd, ttt_linear_dual_slice_maps

    maps_fn = maps_fn or (lambda K_, V_, e_: ttt_linear_dual_slice_maps(
        K_, V_, e_, C=C, eta_scalar=eta_scalar))
    scan_fn = scan_fn or (lambda Q_, K_, V_, e_, w_: ttt_linear_dual_fwd(
        Q_, K_, V_, e_, w_, C=C, eta_scalar=eta_scalar))
    fold_fn = fold_fn or (lambda w0, A_, B_, upto: ttt_dual_state_fold(w0, A_, B_, upto))

    A, B = maps_fn(K, V, eta)
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    both = torch.stack([A, B]).contiguous()
    gathered = torch.empty((world,) + tuple(both.shape), dtype=both.dtype, device=both.device)
    if world > 1:
        dist.all_gather(list(gathered.unbind(0)), both, group=group)
    else:
        gathered[0].copy_(both)
    A_all = gathered[:, 0].contiguous()
    B_all = gathered[:, 1].contiguous()
    start = fold_fn(W0, A_all, B_all, rank)
    O, _ = scan_fn(Q, K, V, eta, start)
    W_final = fold_fn(W0, A_all, B_all, world)
    return O, W_final
