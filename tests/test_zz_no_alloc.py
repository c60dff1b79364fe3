"""The allocation-free In-Place entry point (for callers that cannot allocate device memory,
e.g. runtimes that plan all device buffers up front and refuse allocations while serving) gives
the same results as the workspace entry point, through the C ABI, on consecutive calls that
share its built-in scratch. Collected last so that a failure here cannot hide other tests."""
import ctypes

import pytest
import torch

import weight_linear_attention_ttt_b200 as ttt
from weight_linear_attention_ttt_b200 import inputs as inp

pytestmark = pytest.mark.gpu


def _compare(x, C):
    """Runs the workspace entry point, then the allocation-free one into NaN-filled outputs;
    both run the same kernels on the same inputs, so their results must be bit-identical. The
    allocation-free call must leave the device's free memory and torch's allocation unchanged
    and launch as many kernels as the workspace call."""
    n0 = ttt.launch_count()
    O_ref, W_ref = ttt.inplace_ttt_chunk_fwd(x["Z"], x["Vhat"], x["W0"], x["eta"], C=C)
    launches = ttt.launch_count() - n0
    O = torch.full_like(O_ref, float("nan"))
    W = torch.full_like(W_ref, float("nan"))
    # The first call on a device looks up the scratch array, which loads the part of the library
    # that holds it: the array's memory is taken then (it stays until the process exits). Later
    # calls take nothing.
    ttt.inplace_ttt_chunk_fwd_noalloc(x["Z"], x["Vhat"], x["W0"], x["eta"], C=C, O=O, W_out=W)
    O.fill_(float("nan"))
    W.fill_(float("nan"))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    n0 = ttt.launch_count()
    ttt.inplace_ttt_chunk_fwd_noalloc(x["Z"], x["Vhat"], x["W0"], x["eta"], C=C, O=O, W_out=W)
    torch.cuda.synchronize()
    assert ttt.launch_count() - n0 == launches
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.equal(O, O_ref)
    assert torch.equal(W, W_ref)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(cuda_lib):
    # First call: the larger shape fills more of the shared scratch; the second, smaller call
    # then runs over the first one's leftover contents.
    _compare(inp.inplace_inputs(768, 512, 512, seed=21, device="cuda", eta=1e-2), 256)
    _compare(inp.inplace_inputs(384, 256, 128, seed=22, device="cuda", eta=2e-2), 128)
    assert ttt.read_device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_lib):
    lib = ttt.load_library()
    cap = lib.inplace_ttt_noalloc_max_scratch_bytes()
    assert cap == 32 << 20
    # 4096 x 4096 needs two 32 MiB bf16 copies of W: beyond the built-in scratch.
    need = lib.inplace_ttt_workspace_size(512, 4096, 4096, 256)
    assert need > cap
    n0 = ttt.launch_count()
    v = ctypes.c_void_p
    st = lib.inplace_ttt_chunk_fwd_noalloc(v(1 << 20), v(2 << 20), v(3 << 20),
                                           ctypes.c_float(1e-3), v(4 << 20), v(5 << 20),
                                           512, 4096, 4096, 256, None)
    assert st == 2
    assert b"scratch" in lib.ttt_last_error_message()
    assert lib.ttt_last_error_message().startswith(b"inplace_ttt_chunk_fwd_noalloc")
    # a shape error found by the shared validation names the function the caller used
    st = lib.inplace_ttt_chunk_fwd_noalloc(v(1 << 20), v(2 << 20), v(3 << 20),
                                           ctypes.c_float(1e-3), v(4 << 20), v(5 << 20),
                                           256, 128, 96, 128, None)
    assert st == 2
    assert lib.ttt_last_error_message().startswith(b"inplace_ttt_chunk_fwd_noalloc")
    assert ttt.launch_count() == n0
