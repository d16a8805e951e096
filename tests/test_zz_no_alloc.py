"""flashnorm_proj_noalloc: the projection for callers that cannot allocate.

Some callers must not allocate device memory while they run (runtimes that
pre-plan every byte of the GPU, callers whose framework owns the allocator,
latency-critical loops).  The no-allocation entry point keeps the 1/rms
scratch in a fixed array compiled into the library.  This test calls it
through the C ABI on two calls in a row with different inputs and sizes and
checks each result bit for bit against the allocating entry point,
flashnorm_proj (the same two kernels), and against the fp64 oracle.  The
second call's rows have a 1/rms three orders of magnitude away from the
first's, so a scratch entry left over from the first call cannot go
unnoticed.  It also checks that an M beyond the fixed array is rejected
before any launch.

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
    import oracle
    from parity import frobenius_rel
    lib, f = _noalloc_fn()
    stream = torch.cuda.current_stream().cuda_stream
    # Two calls in a row on different data and sizes.  The second call's rows
    # alternate between N(0,1) and N(0,1) x 1000, so their 1/rms differ from
    # the first call's (~1) by three orders of magnitude: an entry of the
    # shared scratch left over from call 1 would make that row of call 2
    # wrong by a factor of ~1000, not by a few percent.
    for call, (seed, (M, K, N), scale) in enumerate(((0, (1000, 512, 776), False),
                                                     (1, (777, 1024, 264), True))):
        inp = W.make_flashnorm_inputs(seed=seed, M=M, K=K, N=N)
        x_host = inp["x"]
        if scale:
            x_host = x_host.float()
            x_host[1::2] *= 1000.0
            x_host = x_host.to(torch.bfloat16)
        x = x_host.to(DEV)
        Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        st = f(x.data_ptr(), Wf.data_ptr(), y.data_ptr(), M, N, K, 1, inp["eps"], stream)
        assert st == 0, lib.qkn_last_error().decode()
        # the allocating entry point: the same statistics pass and projection
        y_ref = qk.flashnorm_proj(x, Wf, inp["eps"])
        torch.cuda.synchronize()
        same = y.view(torch.int16) == y_ref.view(torch.int16)
        assert bool(same.all()), (f"call {call}: {int((~same).sum())} of {same.numel()} outputs differ from "
                                  f"flashnorm_proj; first rows {torch.nonzero(~same)[:4, 0].tolist()}")
        # and the result itself against the fp64 oracle (original w and W)
        ref = oracle.norm_then_project(x_host, inp["w"], inp["W"], inp["eps"])
        err = frobenius_rel(y, ref)
        assert err <= PROJ_FROB_TOL, f"call {call}: relative Frobenius error {err:.3e} against the oracle"
    assert lib.qkn_check_device(None) == 0, lib.qkn_last_error()


def test_noalloc_at_the_row_limit():
    # exactly as many rows as the fixed scratch holds: every entry of it is written
    # and read, and the result is still the allocating entry point's, bit for bit
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected on a machine without CUDA")
    lib, f = _noalloc_fn()
    M, K, N = MAX_ROWS, 64, 72
    inp = W.make_flashnorm_inputs(seed=9, M=16, K=K, N=N)  # weights; rows drawn below
    g = torch.Generator().manual_seed(10)
    x = (torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g))).to(torch.bfloat16).to(DEV)
    Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = f(x.data_ptr(), Wf.data_ptr(), y.data_ptr(), M, N, K, 1, inp["eps"], torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.qkn_last_error().decode()
    y_ref = qk.flashnorm_proj(x, Wf, inp["eps"])
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert lib.qkn_check_device(None) == 0, lib.qkn_last_error()


def test_noalloc_rejects_rows_beyond_the_fixed_scratch():
    lib, f = _noalloc_fn()
    # validated on the host before anything is launched: pointers are never touched
    st = f(0x10000, 0x10000, 0x10000, MAX_ROWS + 1, 256, 64, 1, 1e-6, None)
    assert st == 2  # QKN_ERR_SHAPE
    assert "fixed scratch" in lib.qkn_last_error().decode()
