"""flashnorm_proj_noalloc: the projection for callers that cannot allocate.

Some callers must not allocate device memory while they run (runtimes that
pre-plan every byte of the GPU, callers whose framework owns the allocator,
latency-critical loops).  The no-allocation entry point keeps the 1/rms
scratch in a fixed array compiled into the library.  This test calls it
through the C ABI and checks it against the allocating entry point,
flashnorm_proj, on two calls in a row with different inputs and sizes (the
second call must not see the first call's scratch), and that an M beyond the
fixed array is rejected before any launch.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import rmsnorm_qknorm_b200 as qk
from parity import PROJ_FROB_TOL
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_ROWS = 262144


def _noalloc_fn():
    lib = qk.load_library()
    f = lib.flashnorm_proj_noalloc
    p, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [p, p, p, i64, i64, i64, ctypes.c_int, ctypes.c_float, p]
    f.restype = ctypes.c_int
    return lib, f


def test_noalloc_matches_allocating_entry_point():
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected on a machine without CUDA")
    lib, f = _noalloc_fn()
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row: a larger problem, then a smaller one on different data
    for seed, (M, K, N) in ((0, (1000, 512, 776)), (1, (257, 1024, 264))):
        inp = W.make_flashnorm_inputs(seed=seed, M=M, K=K, N=N)
        x = inp["x"].to(DEV)
        Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        st = f(x.data_ptr(), Wf.data_ptr(), y.data_ptr(), M, N, K, 1, inp["eps"], stream)
        assert st == 0, lib.qkn_last_error().decode()
        y_ref = qk.flashnorm_proj(x, Wf, inp["eps"])  # the allocating entry point
        torch.cuda.synchronize()
        ref = y_ref.double()
        err = ((y.double() - ref).norm() / ref.norm()).item()
        assert err <= PROJ_FROB_TOL, f"call {seed}: relative Frobenius error {err:.3e}"
    assert lib.qkn_check_device(None) == 0, lib.qkn_last_error()


def test_noalloc_rejects_rows_beyond_the_fixed_scratch():
    lib, f = _noalloc_fn()
    # validated on the host before anything is launched: pointers are never touched
    st = f(0x10000, 0x10000, 0x10000, MAX_ROWS + 1, 256, 64, 1, 1e-6, None)
    assert st == 2  # QKN_ERR_SHAPE
    assert "fixed scratch" in lib.qkn_last_error().decode()
