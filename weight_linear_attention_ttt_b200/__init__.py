"""Python binding of libttt_b200 (the C ABI declared in include/ttt.h).

Argument marshalling only: each function checks torch tensors, allocates missing outputs and
workspace with torch (device memory plumbing), and calls the C entry point of the same name on
the current CUDA stream. Every step of the computation runs in the library's CUDA kernels; there
is no CPU or PyTorch fallback, and a missing library raises at load time.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libttt_b200.so")

TTT_DTYPE_F32 = 0
TTT_DTYPE_BF16 = 1
STATUS = {0: "TTT_OK", 1: "TTT_ERR_INVALID_ARG", 2: "TTT_ERR_UNSUPPORTED",
          3: "TTT_ERR_WORKSPACE", 4: "TTT_ERR_CUDA", 5: "TTT_ERR_TIMEOUT"}

# Every symbol include/ttt.h declares.
EXPORTED_SYMBOLS = (
    "ttt_status_string", "ttt_last_error_message", "ttt_version", "ttt_launch_count",
    "ttt_read_device_error", "ttt_set_tuning", "ttt_get_tuning", "ttt_reset_tuning",
    "ttt_linear_dual_workspace_size", "ttt_linear_dual_fwd",
    "ttt_linear_dual_seg_workspace_size", "ttt_linear_dual_seg_fwd",
    "ttt_assoc_scan_workspace_size", "ttt_assoc_scan_fwd", "ttt_assoc_state_fwd",
    "ttt_assoc_scan_bwd_workspace_size", "ttt_assoc_scan_bwd",
    "ttt_linear_dual_bwd_workspace_size", "ttt_linear_dual_bwd",
    "ttt_linear_dual_seg_bwd_workspace_size", "ttt_linear_dual_seg_bwd",
    "ttt_linear_dual_slice_maps_workspace_size", "ttt_linear_dual_slice_maps",
    "ttt_dual_state_fold",
    "ttt_assoc_momentum_workspace_size", "ttt_assoc_momentum_fwd",
    "ttt_state_prefix_sum",
    "inplace_ttt_workspace_size", "inplace_ttt_chunk_fwd",
    "inplace_ttt_noalloc_max_scratch_bytes", "inplace_ttt_chunk_fwd_noalloc",
    "ttt_lm_target_workspace_size", "ttt_lm_target_fwd",
    "inplace_ttt_lm_workspace_size", "inplace_ttt_lm_chunk_fwd",
)

_LIB: Optional[ctypes.CDLL] = None


class TTTError(RuntimeError):
    """A non-OK status from the library; ``status`` holds the code."""

    def __init__(self, fn: str, status: int, detail: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {detail}")
        self.status = status


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads the CUDA library (once). Raises if it has not been built."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"CUDA extension not built: {p} is missing "
            "(run `python -m weight_linear_attention_ttt_b200.build`)")
    lib = ctypes.CDLL(p)
    c_int, c_float, c_size, vp, fp = (ctypes.c_int, ctypes.c_float, ctypes.c_size_t,
                                      ctypes.c_void_p, ctypes.c_void_p)
    lib.ttt_status_string.restype = ctypes.c_char_p
    lib.ttt_status_string.argtypes = [c_int]
    lib.ttt_last_error_message.restype = ctypes.c_char_p
    lib.ttt_last_error_message.argtypes = []
    lib.ttt_version.restype = c_int
    lib.ttt_launch_count.restype = ctypes.c_uint64
    lib.ttt_read_device_error.restype = c_int
    lib.ttt_read_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    lib.ttt_set_tuning.restype = c_int
    lib.ttt_set_tuning.argtypes = [ctypes.c_char_p, c_int]
    lib.ttt_get_tuning.restype = c_int
    lib.ttt_get_tuning.argtypes = [ctypes.c_char_p]
    lib.ttt_reset_tuning.restype = None
    lib.ttt_reset_tuning.argtypes = []
    state_args = [vp, vp, vp, fp, c_float, fp, vp, fp, c_int, c_int, c_int, c_int, c_int, c_int,
                  vp, c_size, vp]
    for name in ("ttt_linear_dual_fwd", "ttt_assoc_scan_fwd"):
        getattr(lib, name).restype = c_int
        getattr(lib, name).argtypes = state_args
    for name in ("ttt_linear_dual_workspace_size", "ttt_assoc_scan_workspace_size",
                 "ttt_assoc_scan_bwd_workspace_size", "ttt_assoc_momentum_workspace_size",
                 "ttt_linear_dual_bwd_workspace_size"):
        getattr(lib, name).restype = c_size
        getattr(lib, name).argtypes = [c_int] * 6
    for name in ("ttt_assoc_scan_bwd", "ttt_linear_dual_bwd"):
        getattr(lib, name).restype = c_int
        getattr(lib, name).argtypes = [vp, vp, vp, fp, c_float, fp, vp, fp, vp, vp, vp, fp, fp,
                                       c_int, c_int, c_int, c_int, c_int, c_int, vp, c_size, vp]
    lib.ttt_linear_dual_slice_maps_workspace_size.restype = c_size
    lib.ttt_linear_dual_slice_maps_workspace_size.argtypes = [c_int] * 6
    lib.ttt_linear_dual_slice_maps.restype = c_int
    lib.ttt_linear_dual_slice_maps.argtypes = [vp, vp, fp, c_float, fp, fp, c_int, c_int, c_int,
                                               c_int, c_int, c_int, vp, c_size, vp]
    lib.ttt_dual_state_fold.restype = c_int
    lib.ttt_dual_state_fold.argtypes = [fp, fp, fp, c_int, c_int, fp, c_int, c_int, c_int, vp]
    lib.ttt_linear_dual_seg_bwd_workspace_size.restype = c_size
    lib.ttt_linear_dual_seg_bwd_workspace_size.argtypes = [c_int] * 7
    lib.ttt_linear_dual_seg_bwd.restype = c_int
    lib.ttt_linear_dual_seg_bwd.argtypes = [vp, vp, vp, fp, c_float, fp, vp, fp, vp, vp, vp, fp,
                                            fp, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                            vp, c_size, vp]
    lib.ttt_linear_dual_seg_workspace_size.restype = c_size
    lib.ttt_linear_dual_seg_workspace_size.argtypes = [c_int] * 7
    lib.ttt_linear_dual_seg_fwd.restype = c_int
    lib.ttt_linear_dual_seg_fwd.argtypes = [vp, vp, vp, fp, c_float, fp, vp, fp, c_int, c_int,
                                            c_int, c_int, c_int, c_int, c_int, vp, c_size, vp]
    lib.ttt_assoc_momentum_fwd.restype = c_int
    lib.ttt_assoc_momentum_fwd.argtypes = [vp, vp, vp, fp, c_float, c_float, fp, fp, vp, fp, fp,
                                           c_int, c_int, c_int, c_int, c_int, c_int, vp, c_size,
                                           vp]
    lib.ttt_assoc_state_fwd.restype = c_int
    lib.ttt_assoc_state_fwd.argtypes = [vp, vp, fp, c_float, fp, c_int, c_int, c_int, c_int,
                                        c_int, c_int, vp]
    lib.ttt_state_prefix_sum.restype = c_int
    lib.ttt_state_prefix_sum.argtypes = [fp, fp, c_int, c_int, c_int, c_int, c_int, fp, vp]
    lib.inplace_ttt_workspace_size.restype = c_size
    lib.inplace_ttt_workspace_size.argtypes = [c_int] * 4
    lib.inplace_ttt_chunk_fwd.restype = c_int
    lib.inplace_ttt_chunk_fwd.argtypes = [vp, vp, vp, c_float, vp, fp, c_int, c_int, c_int,
                                          c_int, vp, c_size, vp]
    lib.inplace_ttt_noalloc_max_scratch_bytes.restype = c_size
    lib.inplace_ttt_noalloc_max_scratch_bytes.argtypes = []
    lib.inplace_ttt_chunk_fwd_noalloc.restype = c_int
    lib.inplace_ttt_chunk_fwd_noalloc.argtypes = [vp, vp, vp, c_float, vp, fp, c_int, c_int,
                                                  c_int, c_int, vp]
    lib.ttt_lm_target_workspace_size.restype = c_size
    lib.ttt_lm_target_workspace_size.argtypes = [c_int] * 4
    lib.ttt_lm_target_fwd.restype = c_int
    lib.ttt_lm_target_fwd.argtypes = [vp, fp, vp, vp, c_int, c_int, c_int, c_int, vp, c_size, vp]
    lib.inplace_ttt_lm_workspace_size.restype = c_size
    lib.inplace_ttt_lm_workspace_size.argtypes = [c_int] * 6
    lib.inplace_ttt_lm_chunk_fwd.restype = c_int
    lib.inplace_ttt_lm_chunk_fwd.argtypes = [vp, vp, fp, vp, vp, c_float, vp, fp, c_int, c_int,
                                             c_int, c_int, c_int, c_int, vp, c_size, vp]
    if path is None:
        _LIB = lib
    return lib


def _check(fn: str, status: int):
    if status != 0:
        raise TTTError(fn, status, load_library().ttt_last_error_message().decode())


def _stream_ptr(stream):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.float32:
        return TTT_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return TTT_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _require(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _state_call(fn_name: str, ws_name: str, Q, K, V, eta, eta_scalar, S0, C, O, S_out,
                workspace, stream):
    import torch

    lib = load_library()
    _require(Q.dim() == 4, "Q, K, V must be [B, H, T, d]")
    B, H, T, d = Q.shape
    for t in (Q, K, V):
        _require(t.is_cuda and t.is_contiguous() and t.shape == Q.shape and t.dtype == Q.dtype,
                 "Q, K, V must be contiguous CUDA tensors of one shape and dtype")
    dt = _dtype_code(Q)
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    if S0 is not None:
        _require(S0.is_cuda and S0.dtype == torch.float32 and S0.is_contiguous() and
                 tuple(S0.shape) == (B, H, d, d), "initial state must be fp32 [B, H, d, d]")
    if O is None:
        O = torch.empty_like(Q)
    if S_out is None:
        S_out = torch.empty((B, H, d, d), device=Q.device, dtype=torch.float32)
    ws_bytes = getattr(lib, ws_name)(B, H, T, d, C, dt)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=Q.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = getattr(lib, fn_name)(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), ctypes.c_float(eta_scalar),
                               _ptr(S0), _ptr(O), _ptr(S_out), B, H, T, d, C, dt,
                               _ptr(workspace), wsz, _stream_ptr(stream))
    _check(fn_name, st)
    return O, S_out


def ttt_linear_dual_fwd(Q, K, V, eta=None, W0=None, *, C: int, eta_scalar: float = 0.0,
                        O=None, W_out=None, workspace=None, stream=None) -> Tuple:
    """TTT-Linear mini-batch dual form. Returns (O, W_out); see include/ttt.h."""
    return _state_call("ttt_linear_dual_fwd", "ttt_linear_dual_workspace_size", Q, K, V, eta,
                       eta_scalar, W0, C, O, W_out, workspace, stream)


def ttt_linear_dual_seg_fwd(Q, K, V, eta=None, W0=None, *, C: int, segments: int = 0,
                            eta_scalar: float = 0.0, O=None, W_out=None, workspace=None,
                            stream=None) -> Tuple:
    """The dual form evaluated sequence-parallel (segment-affine scan); same results as
    ttt_linear_dual_fwd. segments = 0 picks the count. Returns (O, W_out); see include/ttt.h."""
    import torch

    lib = load_library()
    _require(Q.dim() == 4, "Q, K, V must be [B, H, T, d]")
    B, H, T, d = Q.shape
    for t in (Q, K, V):
        _require(t.is_cuda and t.is_contiguous() and t.shape == Q.shape and t.dtype == Q.dtype,
                 "Q, K, V must be contiguous CUDA tensors of one shape and dtype")
    dt = _dtype_code(Q)
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    if W0 is not None:
        _require(W0.is_cuda and W0.dtype == torch.float32 and W0.is_contiguous() and
                 tuple(W0.shape) == (B, H, d, d), "initial state must be fp32 [B, H, d, d]")
    O = torch.empty_like(Q) if O is None else O
    if W_out is None:
        W_out = torch.empty((B, H, d, d), device=Q.device, dtype=torch.float32)
    ws_bytes = lib.ttt_linear_dual_seg_workspace_size(B, H, T, d, C, dt, segments)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=Q.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.ttt_linear_dual_seg_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta),
                                     ctypes.c_float(eta_scalar), _ptr(W0), _ptr(O), _ptr(W_out),
                                     B, H, T, d, C, dt, segments, _ptr(workspace), wsz,
                                     _stream_ptr(stream))
    _check("ttt_linear_dual_seg_fwd", st)
    return O, W_out


def ttt_assoc_scan_fwd(Q, K, V, eta=None, S0=None, *, C: int, eta_scalar: float = 0.0,
                       O=None, S_out=None, workspace=None, stream=None) -> Tuple:
    """Associative (gradient-ascent) linear-attention mode. Returns (O, S_out)."""
    return _state_call("ttt_assoc_scan_fwd", "ttt_assoc_scan_workspace_size", Q, K, V, eta,
                       eta_scalar, S0, C, O, S_out, workspace, stream)


def ttt_assoc_scan_bwd(Q, K, V, eta, S0, dO, dS_out=None, *, C: int, eta_scalar: float = 0.0,
                       dQ=None, dK=None, dV=None, deta=None, dS0=None, workspace=None,
                       stream=None) -> Tuple:
    """Backward of the associative mode: gradients of a loss whose gradients with respect to the
    forward's O and S_out are dO and dS_out (None: zeros). Returns (dQ, dK, dV, deta, dS0);
    deta is per token even when eta is None (the scalar rate's gradient is its sum)."""
    import torch

    lib = load_library()
    _require(Q.dim() == 4, "Q, K, V, dO must be [B, H, T, d]")
    B, H, T, d = Q.shape
    for t in (Q, K, V, dO):
        _require(t.is_cuda and t.is_contiguous() and t.shape == Q.shape and t.dtype == Q.dtype,
                 "Q, K, V, dO must be contiguous CUDA tensors of one shape and dtype")
    dt = _dtype_code(Q)
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    for t in (S0, dS_out):
        if t is not None:
            _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                     tuple(t.shape) == (B, H, d, d), "states must be fp32 [B, H, d, d]")
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(Q) if dK is None else dK
    dV = torch.empty_like(Q) if dV is None else dV
    if deta is None:
        deta = torch.empty((B, H, T), device=Q.device, dtype=torch.float32)
    if dS0 is None:
        dS0 = torch.empty((B, H, d, d), device=Q.device, dtype=torch.float32)
    ws_bytes = lib.ttt_assoc_scan_bwd_workspace_size(B, H, T, d, C, dt)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=Q.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.ttt_assoc_scan_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), ctypes.c_float(eta_scalar),
                                _ptr(S0), _ptr(dO), _ptr(dS_out), _ptr(dQ), _ptr(dK), _ptr(dV),
                                _ptr(deta), _ptr(dS0), B, H, T, d, C, dt, _ptr(workspace), wsz,
                                _stream_ptr(stream))
    _check("ttt_assoc_scan_bwd", st)
    return dQ, dK, dV, deta, dS0


def ttt_linear_dual_bwd(Q, K, V, eta, W0, dO, dW_out=None, *, C: int, eta_scalar: float = 0.0,
                        dQ=None, dK=None, dV=None, deta=None, dW0=None, workspace=None,
                        stream=None) -> Tuple:
    """Backward of the dual form: gradients of a loss whose gradients with respect to the
    forward's O and W_out are dO and dW_out (None: zeros). Returns (dQ, dK, dV, deta, dW0);
    deta is per token even when eta is None (the scalar rate's gradient is its sum)."""
    import torch

    lib = load_library()
    _require(Q.dim() == 4, "Q, K, V, dO must be [B, H, T, d]")
    B, H, T, d = Q.shape
    for t in (Q, K, V, dO):
        _require(t.is_cuda and t.is_contiguous() and t.shape == Q.shape and t.dtype == Q.dtype,
                 "Q, K, V, dO must be contiguous CUDA tensors of one shape and dtype")
    dt = _dtype_code(Q)
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    for t in (W0, dW_out):
        if t is not None:
            _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                     tuple(t.shape) == (B, H, d, d), "states must be fp32 [B, H, d, d]")
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(Q) if dK is None else dK
    dV = torch.empty_like(Q) if dV is None else dV
    if deta is None:
        deta = torch.empty((B, H, T), device=Q.device, dtype=torch.float32)
    if dW0 is None:
        dW0 = torch.empty((B, H, d, d), device=Q.device, dtype=torch.float32)
    ws_bytes = lib.ttt_linear_dual_bwd_workspace_size(B, H, T, d, C, dt)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=Q.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.ttt_linear_dual_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), ctypes.c_float(eta_scalar),
                                 _ptr(W0), _ptr(dO), _ptr(dW_out), _ptr(dQ), _ptr(dK), _ptr(dV),
                                 _ptr(deta), _ptr(dW0), B, H, T, d, C, dt, _ptr(workspace), wsz,
                                 _stream_ptr(stream))
    _check("ttt_linear_dual_bwd", st)
    return dQ, dK, dV, deta, dW0


def ttt_linear_dual_seg_bwd(Q, K, V, eta, W0, dO, dW_out=None, *, C: int, segments: int = 0,
                            eta_scalar: float = 0.0, dQ=None, dK=None, dV=None, deta=None,
                            dW0=None, workspace=None, stream=None) -> Tuple:
    """ttt_linear_dual_bwd evaluated over segments of each stream (segments = 0 picks the
    count). Returns (dQ, dK, dV, deta, dW0)."""
    import torch

    lib = load_library()
    _require(Q.dim() == 4, "Q, K, V, dO must be [B, H, T, d]")
    B, H, T, d = Q.shape
    for t in (Q, K, V, dO):
        _require(t.is_cuda and t.is_contiguous() and t.shape == Q.shape and t.dtype == Q.dtype,
                 "Q, K, V, dO must be contiguous CUDA tensors of one shape and dtype")
    dt = _dtype_code(Q)
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    for t in (W0, dW_out):
        if t is not None:
            _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                     tuple(t.shape) == (B, H, d, d), "states must be fp32 [B, H, d, d]")
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(Q) if dK is None else dK
    dV = torch.empty_like(Q) if dV is None else dV
    if deta is None:
        deta = torch.empty((B, H, T), device=Q.device, dtype=torch.float32)
    if dW0 is None:
        dW0 = torch.empty((B, H, d, d), device=Q.device, dtype=torch.float32)
    ws_bytes = lib.ttt_linear_dual_seg_bwd_workspace_size(B, H, T, d, C, dt, segments)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=Q.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.ttt_linear_dual_seg_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta),
                                     ctypes.c_float(eta_scalar), _ptr(W0), _ptr(dO),
                                     _ptr(dW_out), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(deta),
                                     _ptr(dW0), B, H, T, d, C, dt, segments, _ptr(workspace),
                                     wsz, _stream_ptr(stream))
    _check("ttt_linear_dual_seg_bwd", st)
    return dQ, dK, dV, deta, dW0


def ttt_linear_dual_slice_maps(K, V, eta=None, *, C: int, eta_scalar: float = 0.0,
                               A_out=None, B_out=None, workspace=None, stream=None) -> Tuple:
    """The affine map W_end = A W_start + B of a token slice of every stream (dual form).
    Returns (A [B,H,d,d], B [B,H,d,d]) fp32."""
    import torch

    lib = load_library()
    _require(K.dim() == 4, "K, V must be [B, H, T, d]")
    B, H, T, d = K.shape
    for t in (K, V):
        _require(t.is_cuda and t.is_contiguous() and t.shape == K.shape and t.dtype == K.dtype,
                 "K, V must be contiguous CUDA tensors of one shape and dtype")
    dt = _dtype_code(K)
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    if A_out is None:
        A_out = torch.empty((B, H, d, d), device=K.device, dtype=torch.float32)
    if B_out is None:
        B_out = torch.empty((B, H, d, d), device=K.device, dtype=torch.float32)
    ws_bytes = lib.ttt_linear_dual_slice_maps_workspace_size(B, H, T, d, C, dt)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=K.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.ttt_linear_dual_slice_maps(_ptr(K), _ptr(V), _ptr(eta), ctypes.c_float(eta_scalar),
                                        _ptr(A_out), _ptr(B_out), B, H, T, d, C, dt,
                                        _ptr(workspace), wsz, _stream_ptr(stream))
    _check("ttt_linear_dual_slice_maps", st)
    return A_out, B_out


def ttt_dual_state_fold(W0, A_maps, B_maps, upto: int, *, W_out=None, stream=None):
    """W_out = maps 0 .. upto-1 of A_maps / B_maps ([n, B, H, d, d] fp32) applied in order to
    W0 ([B, H, d, d] fp32 or None = zeros)."""
    import torch

    lib = load_library()
    _require(A_maps.dim() == 5 and A_maps.shape == B_maps.shape, "maps must be [n, B, H, d, d]")
    n, B, H, d, _ = A_maps.shape
    for t in (A_maps, B_maps):
        _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous(),
                 "maps must be contiguous fp32 CUDA tensors")
    if W0 is not None:
        _require(W0.is_cuda and W0.dtype == torch.float32 and W0.is_contiguous() and
                 tuple(W0.shape) == (B, H, d, d), "W0 must be fp32 [B, H, d, d]")
    if W_out is None:
        W_out = torch.empty((B, H, d, d), device=A_maps.device, dtype=torch.float32)
    st = lib.ttt_dual_state_fold(_ptr(W0), _ptr(A_maps), _ptr(B_maps), n, upto, _ptr(W_out),
                                 B, H, d, _stream_ptr(stream))
    _check("ttt_dual_state_fold", st)
    return W_out


def ttt_assoc_momentum_fwd(Q, K, V, eta, beta: float, S0=None, M0=None, *, C: int,
                           eta_scalar: float = 0.0, O=None, S_out=None, M_out=None,
                           workspace=None, stream=None) -> Tuple:
    """Associative mode with a momentum inner loop (M = beta M + eta k^T v, S += M, o = q S).
    Returns (O, S_out, M_out); see include/ttt.h."""
    import torch

    lib = load_library()
    _require(Q.dim() == 4, "Q, K, V must be [B, H, T, d]")
    B, H, T, d = Q.shape
    for t in (Q, K, V):
        _require(t.is_cuda and t.is_contiguous() and t.shape == Q.shape and t.dtype == Q.dtype,
                 "Q, K, V must be contiguous CUDA tensors of one shape and dtype")
    dt = _dtype_code(Q)
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    for t in (S0, M0):
        if t is not None:
            _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                     tuple(t.shape) == (B, H, d, d), "states must be fp32 [B, H, d, d]")
    O = torch.empty_like(Q) if O is None else O
    if S_out is None:
        S_out = torch.empty((B, H, d, d), device=Q.device, dtype=torch.float32)
    if M_out is None:
        M_out = torch.empty((B, H, d, d), device=Q.device, dtype=torch.float32)
    ws_bytes = lib.ttt_assoc_momentum_workspace_size(B, H, T, d, C, dt)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=Q.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.ttt_assoc_momentum_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta),
                                    ctypes.c_float(eta_scalar), ctypes.c_float(beta), _ptr(S0),
                                    _ptr(M0), _ptr(O), _ptr(S_out), _ptr(M_out), B, H, T, d, C,
                                    dt, _ptr(workspace), wsz, _stream_ptr(stream))
    _check("ttt_assoc_momentum_fwd", st)
    return O, S_out, M_out


def ttt_assoc_state_fwd(K, V, eta=None, *, C: int, eta_scalar: float = 0.0, dS=None,
                        stream=None):
    """State increment of a sequence slice: dS = sum_t eta_t k_t^T v_t. Returns dS."""
    import torch

    lib = load_library()
    _require(K.dim() == 4 and K.shape == V.shape, "K, V must be [B, H, T, d] of one shape")
    for t in (K, V):
        _require(t.is_cuda and t.is_contiguous() and t.dtype == K.dtype,
                 "K, V must be contiguous CUDA tensors of one dtype")
    B, H, T, d = K.shape
    if eta is not None:
        _require(eta.is_cuda and eta.dtype == torch.float32 and eta.is_contiguous() and
                 tuple(eta.shape) == (B, H, T), "eta must be a contiguous fp32 [B, H, T] tensor")
    if dS is None:
        dS = torch.empty((B, H, d, d), device=K.device, dtype=torch.float32)
    st = lib.ttt_assoc_state_fwd(_ptr(K), _ptr(V), _ptr(eta), ctypes.c_float(eta_scalar),
                                 _ptr(dS), B, H, T, d, C, _dtype_code(K), _stream_ptr(stream))
    _check("ttt_assoc_state_fwd", st)
    return dS


def ttt_state_prefix_sum(S0, increments, upto: int, *, out=None, stream=None):
    """out = S0 + sum_{r < upto} increments[r]; increments [R, B, H, d, d] fp32."""
    import torch

    lib = load_library()
    _require(increments.dim() == 5 and increments.dtype == torch.float32 and
             increments.is_cuda and increments.is_contiguous(),
             "increments must be a contiguous fp32 CUDA tensor [R, B, H, d, d]")
    R, B, H, d, _ = increments.shape
    if S0 is not None:
        _require(S0.is_cuda and S0.dtype == torch.float32 and S0.is_contiguous() and
                 tuple(S0.shape) == (B, H, d, d), "S0 must be fp32 [B, H, d, d]")
    if out is None:
        out = torch.empty((B, H, d, d), device=increments.device, dtype=torch.float32)
    st = lib.ttt_state_prefix_sum(_ptr(S0), _ptr(increments), R, upto, B, H, d, _ptr(out),
                                  _stream_ptr(stream))
    _check("ttt_state_prefix_sum", st)
    return out


def inplace_ttt_chunk_fwd(Z, Vhat, W0, eta: float, *, C: int, O=None, W_out=None,
                          workspace=None, stream=None) -> Tuple:
    """In-Place TTT W_down chunk update. Returns (O, W_out)."""
    import torch

    lib = load_library()
    _require(Z.dim() == 2 and Vhat.dim() == 2 and W0.dim() == 2, "Z, Vhat, W0 must be 2-D")
    T, Dff = Z.shape
    D = Vhat.shape[1]
    for t in (Z, Vhat, W0):
        _require(t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16,
                 "Z, Vhat, W0 must be contiguous bf16 CUDA tensors")
    _require(Vhat.shape[0] == T and tuple(W0.shape) == (Dff, D), "shape mismatch")
    if O is None:
        O = torch.empty((T, D), device=Z.device, dtype=torch.bfloat16)
    if W_out is None:
        W_out = torch.empty((Dff, D), device=Z.device, dtype=torch.float32)
    ws_bytes = lib.inplace_ttt_workspace_size(T, Dff, D, C)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=Z.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.inplace_ttt_chunk_fwd(_ptr(Z), _ptr(Vhat), _ptr(W0), ctypes.c_float(eta), _ptr(O),
                                   _ptr(W_out), T, Dff, D, C, _ptr(workspace), wsz,
                                   _stream_ptr(stream))
    _check("inplace_ttt_chunk_fwd", st)
    return O, W_out


def inplace_ttt_chunk_fwd_noalloc(Z, Vhat, W0, eta: float, *, C: int, O=None, W_out=None,
                                  stream=None) -> Tuple:
    """In-Place W_down update through the library's allocation-free entry point: the C call
    takes no workspace (its scratch is a fixed static device array shared by all calls), for
    callers that cannot allocate device memory. Missing outputs are allocated here by torch for
    convenience; pass O and W_out to allocate nothing. Returns (O, W_out)."""
    import torch

    lib = load_library()
    _require(Z.dim() == 2 and Vhat.dim() == 2 and W0.dim() == 2, "Z, Vhat, W0 must be 2-D")
    T, Dff = Z.shape
    D = Vhat.shape[1]
    for t in (Z, Vhat, W0):
        _require(t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16,
                 "Z, Vhat, W0 must be contiguous bf16 CUDA tensors")
    _require(Vhat.shape[0] == T and tuple(W0.shape) == (Dff, D), "shape mismatch")
    if O is None:
        O = torch.empty((T, D), device=Z.device, dtype=torch.bfloat16)
    if W_out is None:
        W_out = torch.empty((Dff, D), device=Z.device, dtype=torch.float32)
    st = lib.inplace_ttt_chunk_fwd_noalloc(_ptr(Z), _ptr(Vhat), _ptr(W0), ctypes.c_float(eta),
                                           _ptr(O), _ptr(W_out), T, Dff, D, C,
                                           _stream_ptr(stream))
    _check("inplace_ttt_chunk_fwd_noalloc", st)
    return O, W_out


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(load_library().ttt_launch_count())


def set_tuning(key: str, value: int) -> None:
    """Selects a kernel variant process-wide (0 = the library's automatic choice); the keys are
    listed with ttt_set_tuning in include/ttt.h."""
    _check("ttt_set_tuning", load_library().ttt_set_tuning(key.encode(), int(value)))


def get_tuning(key: str) -> int:
    return int(load_library().ttt_get_tuning(key.encode()))


def reset_tuning() -> None:
    """Restores every tuning choice to the automatic one."""
    load_library().ttt_reset_tuning()


def read_device_error() -> int:
    """Reads and clears the device error word (synchronous)."""
    v = ctypes.c_uint(0)
    _check("ttt_read_device_error", load_library().ttt_read_device_error(ctypes.byref(v)))
    return int(v.value)


def _lm_checks(X, Wc, Wp):
    import torch

    _require(X.dim() == 2 and X.is_cuda and X.is_contiguous() and X.dtype == torch.bfloat16,
             "X must be a contiguous bf16 [T, Dm] CUDA tensor")
    _require(Wc.dim() == 2 and Wc.is_cuda and Wc.is_contiguous() and Wc.dtype == torch.float32
             and Wc.shape[1] == X.shape[1], "Wc must be a contiguous fp32 [k, Dm] CUDA tensor")
    _require(Wp.dim() == 2 and Wp.is_cuda and Wp.is_contiguous() and Wp.dtype == torch.bfloat16
             and Wp.shape[0] == X.shape[1], "Wp must be a contiguous bf16 [Dm, D] CUDA tensor")


def ttt_lm_target_fwd(X, Wc, Wp, *, Vhat=None, workspace=None, stream=None):
    """LM-aligned target Vhat = conv(X; Wc) Wp (see include/ttt.h). Returns Vhat [T, D] bf16."""
    import torch

    lib = load_library()
    _lm_checks(X, Wc, Wp)
    T, Dm = X.shape
    k, D = Wc.shape[0], Wp.shape[1]
    if Vhat is None:
        Vhat = torch.empty((T, D), device=X.device, dtype=torch.bfloat16)
    nbytes = lib.ttt_lm_target_workspace_size(T, Dm, D, k)
    if workspace is None and nbytes:
        workspace = torch.empty(nbytes, device=X.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.ttt_lm_target_fwd(_ptr(X), _ptr(Wc), _ptr(Wp), _ptr(Vhat), T, Dm, D, k,
                               _ptr(workspace), wsz, _stream_ptr(stream))
    _check("ttt_lm_target_fwd", st)
    return Vhat


def inplace_ttt_lm_chunk_fwd(Z, X, Wc, Wp, W0, eta: float, *, C: int, O=None, W_out=None,
                             workspace=None, stream=None) -> Tuple:
    """In-Place chunk update whose target is the LM-aligned Vhat formed in front of it.
    Returns (O, W_out); see include/ttt.h."""
    import torch

    lib = load_library()
    _lm_checks(X, Wc, Wp)
    _require(Z.dim() == 2 and Z.is_cuda and Z.is_contiguous() and Z.dtype == torch.bfloat16
             and Z.shape[0] == X.shape[0], "Z must be a contiguous bf16 [T, Dff] CUDA tensor")
    T, Dff = Z.shape
    Dm, k, D = X.shape[1], Wc.shape[0], Wp.shape[1]
    _require(tuple(W0.shape) == (Dff, D) and W0.dtype == torch.bfloat16 and W0.is_contiguous(),
             "W0 must be a contiguous bf16 [Dff, D] tensor")
    if O is None:
        O = torch.empty((T, D), device=Z.device, dtype=torch.bfloat16)
    if W_out is None:
        W_out = torch.empty((Dff, D), device=Z.device, dtype=torch.float32)
    nbytes = lib.inplace_ttt_lm_workspace_size(T, Dff, D, Dm, C, k)
    if workspace is None and nbytes:
        workspace = torch.empty(nbytes, device=Z.device, dtype=torch.uint8)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.inplace_ttt_lm_chunk_fwd(_ptr(Z), _ptr(X), _ptr(Wc), _ptr(Wp), _ptr(W0),
                                      ctypes.c_float(eta), _ptr(O), _ptr(W_out), T, Dff, D, Dm,
                                      C, k, _ptr(workspace), wsz, _stream_ptr(stream))
    _check("inplace_ttt_lm_chunk_fwd", st)
    return O, W_out
