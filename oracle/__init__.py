"""fp64 CPU oracle for QK-Norm and FlashNorm -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The CUDA library and its Python binding never
do; the two implementations share no code.

The arithmetic lives in ``qknorm_oracle.c`` (plain fp64 loops, one row at a
time, OpenMP over rows only).  This module compiles it with gcc on first use,
loads it with ctypes and converts arguments: inputs are widened exactly to
float64 (every fp32 and bf16 value is a double), outputs come back as float64
numpy arrays.  Which page passage each function restates is written beside
the C function.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qknorm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-std=c11", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/liboracle.so``; returns the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *GCC_FLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            d, i64, p = ctypes.c_double, ctypes.c_int64, ctypes.c_void_p
            lib.oracle_threads.restype = ctypes.c_int
            lib.oracle_rmsnorm.argtypes = [p, i64, i64, i64, p, d, p]
            lib.oracle_segment_partials.argtypes = [p, i64, i64, i64, i64, p]
            lib.oracle_segment_partials.restype = ctypes.c_int
            lib.oracle_combine_partials.argtypes = [p, i64, i64, p]
            lib.oracle_inv_rms.argtypes = [p, i64, i64, i64, d, p]
            lib.oracle_fold_weights.argtypes = [p, p, i64, i64, p]
            lib.oracle_norm_then_project.argtypes = [p, i64, i64, p, p, i64, d, p]
            lib.oracle_flashnorm_deferred.argtypes = [p, i64, i64, p, i64, d, p]
            lib.oracle_round_bf16.argtypes = [p, i64, p]
            for f in ("oracle_rmsnorm", "oracle_combine_partials", "oracle_inv_rms",
                      "oracle_fold_weights", "oracle_norm_then_project",
                      "oracle_flashnorm_deferred", "oracle_round_bf16"):
                getattr(lib, f).restype = None
            _lib = lib
    return _lib


def as_f64(a) -> np.ndarray:
    """Exact widening of a torch tensor or array (fp32/bf16/f64) to contiguous float64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """OpenMP threads the oracle's loops run on."""
    return int(_load().oracle_threads())


def rmsnorm(x, w, eps: float) -> np.ndarray:
    """RMSNorm of each row of x [rows, d] with weights w [d]; fp64 result."""
    x, w = as_f64(x), as_f64(w)
    rows, d = x.shape
    assert w.shape == (d,)
    y = np.empty((rows, d), dtype=np.float64)
    _load().oracle_rmsnorm(_ptr(x), rows, d, d, _ptr(w), float(eps), _ptr(y))
    return y


def segment_partials(x, n_seg: int) -> np.ndarray:
    """Per-row sums of squares over n_seg contiguous equal segments: [rows, n_seg]."""
    x = as_f64(x)
    rows, d = x.shape
    out = np.empty((rows, n_seg), dtype=np.float64)
    rc = _load().oracle_segment_partials(_ptr(x), rows, d, d, int(n_seg), _ptr(out))
    if rc != 0:
        raise ValueError(f"d={d} is not a multiple of n_seg={n_seg}")
    return out


def combine_partials(partial) -> np.ndarray:
    """Left-to-right combine of [rows, n_seg] partials into the row statistic [rows]."""
    partial = as_f64(partial)
    rows, n_seg = partial.shape
    out = np.empty(rows, dtype=np.float64)
    _load().oracle_combine_partials(_ptr(partial), rows, n_seg, _ptr(out))
    return out


def inv_rms(x, eps: float) -> np.ndarray:
    """1/sqrt(mean(x^2) + eps) for each row of x [rows, d]."""
    x = as_f64(x)
    rows, d = x.shape
    out = np.empty(rows, dtype=np.float64)
    _load().oracle_inv_rms(_ptr(x), rows, d, d, float(eps), _ptr(out))
    return out


def fold_weights(w, W) -> np.ndarray:
    """FlashNorm fold W' = diag(w) W for W [K, N]."""
    w, W = as_f64(w), as_f64(W)
    K, N = W.shape
    assert w.shape == (K,)
    out = np.empty((K, N), dtype=np.float64)
    _load().oracle_fold_weights(_ptr(w), _ptr(W), K, N, _ptr(out))
    return out


def norm_then_project(x, w, W, eps: float) -> np.ndarray:
    """RMSNorm(x; w, eps) @ W, the semantics FlashNorm reformulates: [M, N]."""
    x, w, W = as_f64(x), as_f64(w), as_f64(W)
    M, K = x.shape
    K2, N = W.shape
    assert K == K2 and w.shape == (K,)
    out = np.empty((M, N), dtype=np.float64)
    _load().oracle_norm_then_project(_ptr(x), M, K, _ptr(w), _ptr(W), N, float(eps), _ptr(out))
    return out


def flashnorm_deferred(x, Wf, eps: float) -> np.ndarray:
    """(x @ Wf) / rms(x) with Wf already folded: [M, N]."""
    x, Wf = as_f64(x), as_f64(Wf)
    M, K = x.shape
    K2, N = Wf.shape
    assert K == K2
    out = np.empty((M, N), dtype=np.float64)
    _load().oracle_flashnorm_deferred(_ptr(x), M, K, _ptr(Wf), N, float(eps), _ptr(out))
    return out


def qkv_proj_qknorm(x, w_in, W, wq, wk, nq: int, nk: int, eps: float, eps_qk: float,
                    input_norm: bool = True) -> np.ndarray:
    """Pre-attention path: u = RMSNorm(x; w_in, eps) @ W (or x @ W without the
    input norm), then QK-Norm of the first nq columns (weights wq) and of the
    next nk columns (wk), each over the token's whole slice, eps_qk; the
    remaining columns (v) pass through.  FlashNorm, abstract (norm then
    linear) followed by layerwise QK-Norm (SwiftQK, abstract): [M, N]."""
    W = as_f64(W)
    N = W.shape[1]
    assert 0 < nq and 0 < nk and nq + nk <= N
    u = norm_then_project(x, w_in, W, eps) if input_norm else as_f64(x) @ W  # library matmul as one step
    y = u.copy()
    y[:, :nq] = rmsnorm(np.ascontiguousarray(u[:, :nq]), wq, eps_qk)
    y[:, nq:nq + nk] = rmsnorm(np.ascontiguousarray(u[:, nq:nq + nk]), wk, eps_qk)
    return y


def round_bf16_bits(v) -> np.ndarray:
    """Round-to-nearest-even of float64 values to bfloat16; returns uint16 bit patterns."""
    v = as_f64(v)
    flat = np.ascontiguousarray(v.reshape(-1))
    out = np.empty(flat.shape, dtype=np.uint16)
    _load().oracle_round_bf16(_ptr(flat), flat.size, _ptr(out))
    return out.reshape(v.shape)
