"""C ABI of libqknorm.so on the host (no GPU needed).

* the library builds and loads, and exports every entry point include/*.h declares;
* argument validation returns the documented qkn_status before anything is
  launched (fake, never-dereferenced device addresses are enough for that).
"""
from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

import rmsnorm_qknorm_b200 as qk
from rmsnorm_qknorm_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, NULL, SHAPE, DTYPE, EPS, ALIGN, CUDA, TIMEOUT, UNSUP = range(9)
F32, BF16 = 0, 1
P = 0x10000  # a fake 64 KiB-aligned device address; validation never dereferences it


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(qk.library_path()):
        qbuild.build()
    return qk.load_library()


def declared_symbols() -> list[str]:
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"QKN_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return sorted(set(names))


def test_headers_declare_the_entry_points():
    names = declared_symbols()
    for n in ("qknorm_fused", "rmsnorm_partial_stats", "flashnorm_fold_weights", "flashnorm_proj",
              "qkn_last_error", "qkn_version", "qkn_check_device"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_symbols():
        assert hasattr(lib, n), f"libqknorm.so does not export {n}"


def test_version(lib):
    assert lib.qkn_version().startswith(b"qknorm")


def fused(lib, q=P, k=P, wq=P, wk=P, qo=P, ko=P, T=4, dq=64, dk=64, ldq=None, ldk=None, ldqo=None,
          ldko=None, act=BF16, wdt=BF16, eps=1e-6, n_seg=1):
    ldq = dq if ldq is None else ldq
    ldk = dk if ldk is None else ldk
    ldqo = dq if ldqo is None else ldqo
    ldko = dk if ldko is None else ldko
    return lib.qknorm_fused(q, k, wq, wk, qo, ko, T, dq, dk, ldq, ldk, ldqo, ldko, act, wdt, eps, n_seg,
                            None)


def test_qknorm_validation(lib):
    assert fused(lib, q=None) == NULL
    assert fused(lib, wq=None) == NULL
    assert fused(lib, k=None) == NULL          # dk > 0 but k missing
    assert fused(lib, wk=None) == NULL
    assert "wk" in lib.qkn_last_error().decode()
    assert fused(lib, T=-1) == SHAPE
    assert fused(lib, dq=0) == SHAPE
    assert fused(lib, ldq=32) == SHAPE         # pitch < width
    assert fused(lib, ldqo=16) == SHAPE
    assert fused(lib, n_seg=0) == SHAPE
    assert fused(lib, n_seg=65) == SHAPE       # > QKN_MAX_SEG
    assert fused(lib, dq=60, n_seg=8) == SHAPE  # dq % n_seg
    assert fused(lib, dk=36, n_seg=8) == SHAPE
    assert fused(lib, act=2) == DTYPE
    assert fused(lib, wdt=-1) == DTYPE
    assert fused(lib, eps=-1e-6) == EPS
    assert fused(lib, eps=float("nan")) == EPS
    assert fused(lib, eps=float("inf")) == EPS
    assert fused(lib, q=P + 1) == ALIGN        # not element aligned
    assert fused(lib, act=F32, k=P + 2) == ALIGN
    assert fused(lib, wdt=F32, wq=P + 2) == ALIGN


def test_qknorm_empty_problem_launches_nothing(lib):
    # T == 0 is valid and returns before any CUDA call (works without a GPU)
    assert fused(lib, T=0) == OK
    assert fused(lib, T=0, k=None, wk=None, ko=None, dk=0) == OK
    assert fused(lib, T=0, qo=None, ko=None) == OK  # in place
    assert fused(lib, T=0, q=None, k=None, wq=None, wk=None, qo=None, ko=None) == OK  # empty tensors
    assert fused(lib, T=0, n_seg=3) == SHAPE  # sizes are still validated


def test_partial_stats_validation(lib):
    f = lib.rmsnorm_partial_stats
    assert f(None, 4, 64, 64, BF16, 4, P, None) == NULL
    assert f(P, 4, 64, 64, BF16, 4, None, None) == NULL
    assert f(P, -1, 64, 64, BF16, 4, P, None) == SHAPE
    assert f(P, 4, 64, 32, BF16, 4, P, None) == SHAPE
    assert f(P, 4, 66, 66, BF16, 4, P, None) == SHAPE
    assert f(P, 4, 64, 64, 7, 4, P, None) == DTYPE
    assert f(P, 4, 64, 64, BF16, 4, P + 2, None) == ALIGN
    assert f(P, 0, 64, 64, BF16, 4, P, None) == OK
    assert f(None, 0, 64, 64, BF16, 4, None, None) == OK


def test_fold_validation(lib):
    f = lib.flashnorm_fold_weights
    assert f(None, P, P, 8, 8, BF16, 1, None) == NULL
    assert f(P, P, None, 8, 8, BF16, 1, None) == NULL
    assert f(P, P, P, -8, 8, BF16, 1, None) == SHAPE
    assert f(P, P, P, 8, 8, 5, 1, None) == DTYPE
    assert f(P + 2, P, P, 8, 8, F32, 1, None) == ALIGN
    assert f(P, P, P, 0, 8, BF16, 1, None) == OK


def test_proj_validation(lib):
    f = lib.flashnorm_proj
    assert f(None, P, P, 128, 256, 64, 1, 1e-6, None, None, None) == NULL
    assert f(P, P, P, 0, 256, 64, 1, 1e-6, None, None, None) == SHAPE
    assert f(P, P, P, 128, 250, 64, 1, 1e-6, None, None, None) == SHAPE   # N % 8
    assert f(P, P, P, 128, 256, 60, 1, 1e-6, None, None, None) == SHAPE   # K % 8
    assert f(P, P, P, 128, 256, 64, 0, -1.0, None, None, None) == EPS     # row-major W' is validated too
    # the no-allocation form cannot make the K-major copy a row-major W' needs
    g = lib.flashnorm_proj_noalloc
    g.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_int, ctypes.c_float, ctypes.c_void_p]
    assert g(P, P, P, 128, 256, 64, 0, 1e-6, None) == UNSUP
    assert f(P, P, P, 128, 256, 64, 1, -1.0, None, None, None) == EPS
    assert f(P + 8, P, P, 128, 256, 64, 1, 1e-6, None, None, None) == ALIGN  # TMA needs 16 B
    assert "16-byte" in lib.qkn_last_error().decode()


def test_inv_rms_validation(lib):
    f = lib.flashnorm_inv_rms
    assert f(None, P, 4, 64, 1e-6, None) == NULL
    assert f(P, None, 4, 64, 1e-6, None) == NULL
    assert f(P, P, -1, 64, 1e-6, None) == SHAPE
    assert f(P, P, 4, 60, 1e-6, None) == SHAPE     # K % 8
    assert f(P, P, 4, 64, -1.0, None) == EPS
    assert f(P + 8, P, 4, 64, 1e-6, None) == ALIGN  # 16-byte rows
    assert f(None, None, 0, 64, 1e-6, None) == OK   # nothing to do: pointers unused


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    w = torch.ones(64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        qk.qknorm_fused(x, None, w, None)


def test_apply_partials_validation(lib):
    f = lib.rmsnorm_apply_partials
    # (x, w, y, rows, d, ld, ld_out, partial, n_part, prs, ps, d_full, act, wdt, eps, stream)
    assert f(None, P, P, 4, 64, 64, 64, P, 8, 8, 1, 512, BF16, BF16, 1e-6, None) == NULL
    assert f(P, P, P, 4, 64, 32, 64, P, 8, 8, 1, 512, BF16, BF16, 1e-6, None) == SHAPE  # ld < d
    assert f(P, P, P, 4, 64, 64, 64, P, 8, 8, 1, 32, BF16, BF16, 1e-6, None) == SHAPE   # d_full < d
    assert f(P, P, P, 4, 64, 64, 64, P, 0, 8, 1, 512, BF16, BF16, 1e-6, None) == SHAPE  # n_part
    assert f(P, P, P, 4, 64, 64, 64, P, 8, 8, 1, 512, 9, BF16, 1e-6, None) == DTYPE
    assert f(P, P, P, 4, 64, 64, 64, P, 8, 8, 1, 512, BF16, BF16, -1.0, None) == EPS
    assert f(P, P, P, 4, 64, 64, 64, P + 2, 8, 8, 1, 512, BF16, BF16, 1e-6, None) == ALIGN
    assert f(None, None, None, 0, 64, 64, 64, None, 8, 8, 1, 512, BF16, BF16, 1e-6, None) == OK


def test_qkv_norm_proj_validation(lib):
    f = lib.qkv_norm_proj
    # (x, Wf, y, M, K, nq, nk, nv, wq, wk, wv, wdt, eps, n_seg, stream)
    assert f(P, P, P, 8, 64, 64, 32, 32, P, P, None, BF16, 1e-6, 1, None) == NULL     # wv with nv > 0
    assert f(P, P, P, 8, 60, 64, 32, 32, P, P, P, BF16, 1e-6, 1, None) == SHAPE       # K % 8
    assert f(P, P, P, 8, 64, 64, 32, 30, P, P, P, BF16, 1e-6, 1, None) == SHAPE       # N % 8
    assert f(P, P, P, 8, 64, 64, 32, 32, P, P, P, BF16, 1e-6, 3, None) == SHAPE       # n_seg
    assert f(P, P, P, 8, 64, 64, 32, 32, P, P, P, BF16, float("nan"), 1, None) == EPS
    assert f(P + 8, P, P, 8, 64, 64, 32, 32, P, P, P, BF16, 1e-6, 1, None) == ALIGN


def test_fault_hook_validation(lib):
    lib.qkn_testing_arm_wait_fault.argtypes = [ctypes.c_uint64]
    assert lib.qkn_testing_arm_wait_fault(0) == SHAPE
    assert lib.qkn_testing_arm_wait_fault(3_000_000_000) == SHAPE


def test_host_entry_validation(lib):
    # qknorm_fused_host(q, k, wq, wk, q_out, k_out, T, dq, dk, act, wdt, eps, n_seg, ws, ws_bytes, stream)
    f = lib.qknorm_fused_host
    big = 1 << 20

    def h(q=P, k=P, wq=P, wk=P, qo=P, ko=P, T=4, dq=64, dk=64, act=BF16, wdt=BF16, eps=1e-6, n_seg=1,
          ws=P, nbytes=big):
        return f(q, k, wq, wk, qo, ko, T, dq, dk, act, wdt, eps, n_seg, ws, nbytes, None)

    assert h(ws=None) == NULL
    assert h(k=None) == NULL
    assert h(T=-1) == SHAPE
    assert h(dq=60, n_seg=8) == SHAPE
    assert h(act=5) == DTYPE
    assert h(eps=float("nan")) == EPS
    assert h(nbytes=3 * 255) == SHAPE          # not even one row per stream buffer
    assert "workspace" in lib.qkn_last_error().decode()
    assert h(ws=P + 16) == ALIGN               # workspace must be 256-byte aligned
    assert h(T=0, q=None, k=None, qo=None, ko=None, ws=None) == OK


def test_qkv_proj_qknorm_validation(lib):
    # (x, Wf, y, M, K, nq, nk, nv, wq, wk, wdt, eps, eps_qk, inv, inv_out, ws, ws_bytes, stream)
    f = lib.qkv_proj_qknorm

    def c(x=P, Wf=P, y=P, M=8, K=64, nq=64, nk=32, nv=32, wq=P, wk=P, wdt=BF16, eps=1e-6, eps_qk=1e-6,
          inv=None, inv_out=None, ws=None, nbytes=0):
        return f(x, Wf, y, M, K, nq, nk, nv, wq, wk, wdt, eps, eps_qk, inv, inv_out, ws, nbytes, None)

    assert c(wk=None) == NULL
    assert c(y=None) == NULL
    assert c(M=0) == SHAPE
    assert c(nq=0) == SHAPE
    assert c(nv=-8) == SHAPE
    assert c(K=60) == SHAPE
    assert c(nk=36) == SHAPE
    assert c(wdt=7) == DTYPE
    assert c(eps_qk=-1.0) == EPS
    assert c(eps=float("nan"), inv_out=P) == EPS    # eps is used by the statistics pass
    assert c(x=P + 8) == ALIGN
    assert c(wq=P + 4) == ALIGN
    assert c(ws=P + 8, nbytes=1 << 20) == ALIGN
    need = lib.qkv_proj_qknorm_workspace_bytes(8, 64, 32, 32)
    assert need > 0
    assert c(ws=P, nbytes=need - 1) == SHAPE
    assert "workspace" in lib.qkn_last_error().decode()
    assert lib.qkv_proj_qknorm_workspace_bytes(0, 64, 32, 32) == 0


def test_exchange_fault_hook_validation(lib):
    lib.qkn_testing_arm_exchange_fault.argtypes = [ctypes.c_uint64]
    assert lib.qkn_testing_arm_exchange_fault(0) == SHAPE
    assert lib.qkn_testing_arm_exchange_fault(3_000_000_000) == SHAPE
