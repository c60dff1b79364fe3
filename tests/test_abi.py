"""The C-ABI library builds, loads and exports every declared symbol; host-side validation
returns its status before anything is launched (CPU only: no compute call is made)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

import weight_linear_attention_ttt_b200 as ttt
from weight_linear_attention_ttt_b200 import build as ttt_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ttt_build.build()
    return ttt.load_library()


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M):
            if m.group(1) not in ("if", "defined"):
                names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_binding_symbols():
    assert set(_declared_functions()) == set(ttt.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", ttt.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in _declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings_and_version(lib):
    assert lib.ttt_status_string(0) == b"TTT_OK"
    assert lib.ttt_status_string(3) == b"TTT_ERR_WORKSPACE"
    assert lib.ttt_status_string(99) == b"TTT_ERR_UNKNOWN"
    assert lib.ttt_version() >= 10000
    assert lib.ttt_launch_count() == 0  # nothing launched on a CPU-only host


# Fake, never-dereferenced device addresses: validation fails before any CUDA call.
A = 1 << 20


def _dual(lib, **kw):
    args = dict(Q=A, K=2 * A, V=3 * A, eta=4 * A, eta_scalar=0.0, W0=5 * A, O=6 * A, W_out=7 * A,
                B=1, H=1, T=64, d=64, C=16, dt=1, ws=0, ws_bytes=0, stream=0)
    args.update(kw)
    v = ctypes.c_void_p
    return lib.ttt_linear_dual_fwd(v(args["Q"]), v(args["K"]), v(args["V"]), v(args["eta"]),
                                   ctypes.c_float(args["eta_scalar"]), v(args["W0"]),
                                   v(args["O"]), v(args["W_out"]), args["B"], args["H"],
                                   args["T"], args["d"], args["C"], args["dt"], v(args["ws"]),
                                   args["ws_bytes"], v(args["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(Q=0), 1), (dict(O=0), 1), (dict(W_out=0), 1),
    (dict(K=2 * A + 8), 1),                  # misaligned
    (dict(T=60), 1),                         # T % C != 0
    (dict(B=0), 1), (dict(C=-16), 1), (dict(dt=7), 1),
    (dict(d=48), 2), (dict(C=128, T=128), 2),
    (dict(O=A + 64), 1),                     # O overlaps Q
    (dict(W_out=5 * A + 64), 1),             # partial overlap with W0
])
def test_dual_validation(lib, kw, status):
    assert _dual(lib, **kw) == status
    assert lib.ttt_last_error_message() != b""
    assert lib.ttt_launch_count() == 0


def test_assoc_and_inplace_validation(lib):
    v = ctypes.c_void_p
    st = lib.ttt_assoc_scan_fwd(v(A), v(2 * A), v(3 * A), None, ctypes.c_float(1.0), None,
                                v(6 * A), v(7 * A), 1, 1, 100, 128, 64, 1, None, 0, None)
    assert st == 1  # T % C
    st = lib.inplace_ttt_chunk_fwd(v(A), v(2 * A), v(3 * A), ctypes.c_float(1e-3), v(4 * A),
                                   None, 2048, 256, 256, 1024, None, 0, None)
    assert st == 1  # W_out null
    st = lib.inplace_ttt_chunk_fwd(v(A), v(2 * A), v(3 * A), ctypes.c_float(1e-3), v(4 * A),
                                   v(5 * A), 2000, 256, 256, 1024, None, 0, None)
    assert st == 1  # T % C
    assert lib.ttt_launch_count() == 0


def test_python_binding_rejects_non_cuda_tensors(lib):
    import torch

    x = torch.zeros(1, 1, 16, 32)
    with pytest.raises(ValueError):
        ttt.ttt_linear_dual_fwd(x, x, x, C=16)


def _bwd(lib, fn, **kw):
    """Backward entry points (associative and dual form) share one argument list."""
    args = dict(Q=A, K=2 * A, V=3 * A, eta=4 * A, eta_scalar=0.0, S0=5 * A, dO=6 * A,
                dS_out=7 * A, dQ=8 * A, dK=9 * A, dV=10 * A, deta=11 * A, dS0=12 * A,
                B=1, H=1, T=64, d=128, C=64, dt=1, ws=13 * A, ws_bytes=1 << 19, stream=0)
    args.update(kw)
    v = ctypes.c_void_p
    return getattr(lib, fn)(
        v(args["Q"]), v(args["K"]), v(args["V"]), v(args["eta"]),
        ctypes.c_float(args["eta_scalar"]), v(args["S0"]), v(args["dO"]), v(args["dS_out"]),
        v(args["dQ"]), v(args["dK"]), v(args["dV"]), v(args["deta"]), v(args["dS0"]),
        args["B"], args["H"], args["T"], args["d"], args["C"], args["dt"], v(args["ws"]),
        args["ws_bytes"], v(args["stream"]))


@pytest.mark.parametrize("fn,base", [
    ("ttt_assoc_scan_bwd", dict(d=128, C=64, T=128)),
    ("ttt_linear_dual_bwd", dict(d=64, C=16, T=64)),
])
@pytest.mark.parametrize("kw,status", [
    (dict(dQ=0), 1), (dict(dO=0), 1), (dict(deta=0), 1),
    (dict(V=3 * A + 8), 1),                  # misaligned
    (dict(T=100), 1),                        # T % C != 0
    (dict(H=0), 1), (dict(dt=5), 1),
    (dict(d=48), 2),                         # unsupported head dim
    (dict(ws_bytes=16), 3),                  # workspace too small
    (dict(ws=0), 3),
    (dict(dK=2 * A), 1),                     # an output on an input
    (dict(dQ=8 * A, dK=8 * A + 64), 1),      # two outputs overlap
])
def test_backward_validation(lib, fn, base, kw, status):
    ws = {"ws_bytes": 1 << 30}
    assert _bwd(lib, fn, **dict(base, **dict(ws, **kw))) == status
    assert lib.ttt_last_error_message() != b""
    assert lib.ttt_launch_count() == 0


def test_backward_chunk_size_rules(lib):
    # the dual form's backward runs the C = 16 mini-batch only; the associative one any C of
    # 16, 32, 64 on 64-token tiles (T % 64 == 0), and no other head dim than 64 or 128
    assert _bwd(lib, "ttt_linear_dual_bwd", d=64, C=32, T=64, ws_bytes=1 << 30) == 2
    assert _bwd(lib, "ttt_assoc_scan_bwd", d=128, C=16, T=48, ws_bytes=1 << 30) == 2
    assert _bwd(lib, "ttt_assoc_scan_bwd", d=128, C=8, T=64, ws_bytes=1 << 30) == 2
    assert _bwd(lib, "ttt_assoc_scan_bwd", d=96, C=64, T=64, ws_bytes=1 << 30) == 2
    assert lib.ttt_launch_count() == 0


def test_workspace_size_queries(lib):
    # dual-form backward: one bf16 d x d checkpoint per chunk and stream
    assert lib.ttt_linear_dual_bwd_workspace_size(8, 12, 2048, 64, 16, 1) == 8 * 12 * 128 * 64 * 64 * 2
    assert lib.ttt_linear_dual_bwd_workspace_size(8, 12, 2048, 64, 32, 1) == 0   # C unsupported
    assert lib.ttt_linear_dual_bwd_workspace_size(8, 12, 2040, 64, 16, 1) == 0   # T % C
    assert lib.ttt_linear_dual_bwd_workspace_size(1, 1, 64, 64, 16, 0) == 0      # fp32
    assert lib.ttt_assoc_scan_bwd_workspace_size(4, 16, 65536, 128, 64, 1) > 0
    assert lib.ttt_assoc_scan_bwd_workspace_size(4, 16, 65536, 64, 16, 1) > 0
    assert lib.ttt_assoc_scan_bwd_workspace_size(4, 16, 65536, 96, 64, 1) == 0
    assert lib.ttt_assoc_scan_workspace_size(4, 16, 65536 + 32, 128, 32, 1) == 0   # T % 64
    assert lib.ttt_assoc_momentum_workspace_size(4, 16, 65536, 128, 64, 1) > 0
    assert lib.ttt_assoc_momentum_workspace_size(4, 16, 100, 128, 64, 1) == 0
    # the convolved embeddings (bf16, 256-byte aligned) and one 256-byte counter slot
    assert lib.ttt_lm_target_workspace_size(32768, 2560, 2560, 4) == 32768 * 2560 * 2 + 256
    assert lib.ttt_lm_target_workspace_size(0, 2560, 2560, 4) == 0


def test_momentum_validation(lib):
    v = ctypes.c_void_p

    def mom(beta, M_out=9 * A, d=128):
        return lib.ttt_assoc_momentum_fwd(v(A), v(2 * A), v(3 * A), None, ctypes.c_float(1.0),
                                          ctypes.c_float(beta), None, None, v(6 * A), v(7 * A),
                                          v(M_out), 1, 1, 128, d, 64, 1, v(10 * A), 1 << 30, None)

    assert mom(-0.1) == 2 and mom(1.5) == 2 and mom(float("nan")) == 2   # outside [0, 1]
    assert lib.ttt_set_tuning(b"momentum_form", 1) == 0                 # the two-pass form
    assert mom(0.95) == 2 and mom(0.1) == 2 and mom(1.0) == 2          # outside [0.25, 0.9]
    lib.ttt_reset_tuning()
    assert mom(0.5, M_out=0) == 1
    assert mom(0.5, d=96) == 2
    assert mom(0.5, M_out=6 * A + 64) == 1                      # M_out overlaps O
    assert lib.ttt_launch_count() == 0


def test_segmented_entry_points_validation(lib):
    v = ctypes.c_void_p

    def fwd(segments, T=1024, d=64, ws=10 * A, ws_bytes=1 << 30, O=6 * A):
        return lib.ttt_linear_dual_seg_fwd(v(A), v(2 * A), v(3 * A), v(4 * A),
                                           ctypes.c_float(0.0), v(5 * A), v(O), v(7 * A), 1, 1,
                                           T, d, 16, 1, segments, v(ws), ws_bytes, None)

    assert fwd(3) == 1              # 3 does not divide the 64 chunks
    assert fwd(-1) == 1
    assert fwd(4, d=48) == 2
    assert fwd(4, ws_bytes=16) == 3
    assert fwd(4, ws=0) == 3
    assert fwd(4, O=A + 64) == 1    # O overlaps Q
    # sizes: 5 fp32 d x d states per segment (forward); none when one segment is chosen
    assert lib.ttt_linear_dual_seg_workspace_size(1, 1, 1024, 64, 16, 1, 4) == 5 * 4 * 64 * 64 * 4
    assert lib.ttt_linear_dual_seg_workspace_size(1, 1, 1024, 64, 16, 1, 3) == 0
    assert lib.ttt_linear_dual_seg_workspace_size(8, 12, 1024, 64, 16, 1, 0) == 0
    assert lib.ttt_linear_dual_seg_bwd_workspace_size(1, 1, 1024, 64, 16, 1, 4) > \
        lib.ttt_linear_dual_bwd_workspace_size(1, 1, 1024, 64, 16, 1)
    assert lib.ttt_launch_count() == 0


def test_segmented_backward_validation(lib):
    v = ctypes.c_void_p

    def bwd(segments, ws_bytes=1 << 30, dQ=8 * A, d=64):
        return lib.ttt_linear_dual_seg_bwd(v(A), v(2 * A), v(3 * A), v(4 * A),
                                           ctypes.c_float(0.0), v(5 * A), v(6 * A), v(7 * A),
                                           v(dQ), v(9 * A), v(10 * A), v(11 * A), v(12 * A),
                                           1, 1, 1024, d, 16, 1, segments, v(13 * A), ws_bytes,
                                           None)

    assert bwd(3) == 1 and bwd(-2) == 1
    assert bwd(4, d=48) == 2
    assert bwd(4, ws_bytes=16) == 3
    assert bwd(4, dQ=2 * A) == 1    # an output on an input
    assert bwd(4, dQ=0) == 1
    assert lib.ttt_launch_count() == 0


def test_dual_context_parallel_pieces_validation(lib):
    v = ctypes.c_void_p

    def maps(**kw):
        a = dict(K=A, V=2 * A, eta=3 * A, Aout=4 * A, Bout=5 * A, T=256, d=64, C=16, dt=1,
                 ws=6 * A, ws_bytes=1 << 30)
        a.update(kw)
        return lib.ttt_linear_dual_slice_maps(v(a["K"]), v(a["V"]), v(a["eta"]),
                                              ctypes.c_float(0.0), v(a["Aout"]), v(a["Bout"]),
                                              1, 1, a["T"], a["d"], a["C"], a["dt"], v(a["ws"]),
                                              a["ws_bytes"], None)

    assert maps(Bout=0) == 1 and maps(T=250) == 1 and maps(d=48) == 2
    assert maps(ws_bytes=16) == 3 and maps(Aout=A + 64) == 1 and maps(Bout=4 * A + 256) == 1
    need = lib.ttt_linear_dual_slice_maps_workspace_size(1, 1, 256, 64, 16, 1)
    assert need == 256 * 64 * 2 + 64 * 64 * 4

    def fold(**kw):
        a = dict(W0=A, Am=2 * A, Bm=3 * A, n=4, upto=2, Wout=4 * A, d=64)
        a.update(kw)
        return lib.ttt_dual_state_fold(v(a["W0"]), v(a["Am"]), v(a["Bm"]), a["n"], a["upto"],
                                       v(a["Wout"]), 1, 1, a["d"], None)

    assert fold(upto=5) == 1 and fold(upto=-1) == 1 and fold(n=0) == 1 and fold(Am=0) == 1
    assert fold(d=48) == 2 and fold(Wout=2 * A + 64) == 1 and fold(Wout=A + 64) == 1
    assert lib.ttt_launch_count() == 0


def test_tuning_choices_set_get_reset(lib):
    """Kernel-variant choices are explicit library state (nothing is read from the
    environment): unknown keys and negative values are refused, reset restores 0."""
    try:
        assert lib.ttt_get_tuning(b"dual_kernel") == 0
        assert lib.ttt_set_tuning(b"dual_kernel", 3) == 0
        assert lib.ttt_get_tuning(b"dual_kernel") == 3
        assert lib.ttt_set_tuning(b"assoc_parts", 4) == 0
        assert lib.ttt_set_tuning(b"no_such_key", 1) == 1
        assert b"unknown key" in lib.ttt_last_error_message()
        assert lib.ttt_set_tuning(b"dual_column_split", -1) == 1
        assert lib.ttt_get_tuning(b"no_such_key") == -1
        lib.ttt_reset_tuning()
        for key in (b"dual_column_split", b"dual_kernel", b"dual_warp_cols",
                    b"dual_stage_chunks", b"assoc_parts", b"wait_limit_ns",
                    b"inplace_chunks_per_launch", b"dual_cluster_streams"):
            assert lib.ttt_get_tuning(key) == 0
    finally:
        lib.ttt_reset_tuning()


def test_library_reads_no_environment():
    """No kernel variant or tuning choice comes from environment variables."""
    src = glob.glob(os.path.join(ROOT, "weight_linear_attention_ttt_b200", "csrc", "*"))
    for f in src:
        assert "getenv" not in open(f, encoding="utf-8").read(), f
