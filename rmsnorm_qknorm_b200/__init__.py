"""B200-native layerwise QK-Norm and FlashNorm: Python binding of libqknorm.so.

This module only marshals arguments: it checks tensor placement, reads
pointers, pitches and the current CUDA stream from torch, and calls the C ABI
declared in ``include/qknorm.h``.  Every step of the computation runs in the
library's sm_100a kernels; there is no CPU or PyTorch fallback, and a missing
library raises instead of degrading.

Entry points (same names as the C ABI):

* :func:`qknorm_fused` -- RMSNorm of every query row and key row (one launch for
  both wherever their kernels agree),
  statistics built from ``n_seg`` per-segment scalar partial sums combined in a
  fixed order (SwiftQK's tensor-parallel statistic, emulated on one GPU).
* :func:`rmsnorm_partial_stats` -- those per-segment partial sums on their own.
* :func:`flashnorm_fold_weights` -- FlashNorm's W' = diag(w) W.
* :func:`flashnorm_proj` -- y = (x W') * 1/rms(x), the deferred-normalisation
  GEMM with the scaling in the epilogue.
* :func:`rmsnorm_apply_partials` -- the apply step of tensor-parallel QK-Norm:
  normalise a shard from the gathered per-shard partial sums.
* :func:`qkv_norm_proj` -- QKV projection + QKV-normalisation with the
  pre-attention RMSNorm eliminated (FlashNorm's scale-invariance identity).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "QKNormError",
    "load_library",
    "library_path",
    "qknorm_fused",
    "qknorm_fused_host",
    "qkv_proj_qknorm",
    "qkv_proj_qknorm_workspace_bytes",
    "rmsnorm_partial_stats",
    "flashnorm_fold_weights",
    "flashnorm_proj",
    "flashnorm_inv_rms",
    "rmsnorm_apply_partials",
    "qkv_norm_proj",
    "STATUS_NAMES",
    "QKN_MAX_SEG",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libqknorm.so")
_lock = threading.Lock()
_lib = None

QKN_MAX_SEG = 64
QKN_F32, QKN_BF16 = 0, 1
STATUS_NAMES = {
    0: "QKN_OK", 1: "QKN_ERR_NULL", 2: "QKN_ERR_SHAPE", 3: "QKN_ERR_DTYPE", 4: "QKN_ERR_EPS",
    5: "QKN_ERR_ALIGN", 6: "QKN_ERR_CUDA", 7: "QKN_ERR_TIMEOUT", 8: "QKN_ERR_UNSUPPORTED",
}


class QKNormError(RuntimeError):
    """A nonzero qkn_status from the library, with its message."""

    def __init__(self, fn: str, status: int, message: str):
        self.status = status
        self.status_name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{fn}: {self.status_name}: {message}")


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libqknorm.so (built by ``python -m rmsnorm_qknorm_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError(
                f"{_LIB_PATH} is missing: build it with `python -m rmsnorm_qknorm_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(_LIB_PATH)
        p, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        lib.qknorm_fused.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, i64, i64, i64,
                                     i32, i32, f32, i32, p]
        lib.rmsnorm_partial_stats.argtypes = [p, i64, i64, i64, i32, i32, p, p]
        lib.flashnorm_fold_weights.argtypes = [p, p, p, i64, i64, i32, i32, p]
        lib.flashnorm_proj.argtypes = [p, p, p, i64, i64, i64, i32, f32, p, p, p]
        lib.rmsnorm_apply_partials.argtypes = [p, p, p, i64, i64, i64, i64, p, i32, i64, i64, i64,
                                               i32, i32, f32, p]
        lib.qkv_norm_proj.argtypes = [p, p, p, i64, i64, i64, i64, i64, p, p, p, i32, f32, i32, p]
        lib.qknorm_fused_host.argtypes = [p, p, p, p, p, p, i64, i64, i64, i32, i32, f32, i32,
                                          p, ctypes.c_size_t, p]
        lib.qkv_proj_qknorm.argtypes = [p, p, p, i64, i64, i64, i64, i64, p, p, i32, f32, f32, p, p,
                                        p, ctypes.c_size_t, p]
        lib.qkv_proj_qknorm_workspace_bytes.argtypes = [i64, i64, i64, i64]
        lib.qkv_proj_qknorm_workspace_bytes.restype = ctypes.c_size_t
        lib.flashnorm_inv_rms.argtypes = [p, p, i64, i64, f32, p]
        lib.qkn_check_device.argtypes = [p]
        for f in ("qknorm_fused", "qknorm_fused_host", "qkv_proj_qknorm", "rmsnorm_partial_stats", "flashnorm_fold_weights",
                  "flashnorm_proj", "flashnorm_inv_rms", "rmsnorm_apply_partials", "qkv_norm_proj", "qkn_check_device"):
            getattr(lib, f).restype = ctypes.c_int
        lib.qkn_last_error.restype = ctypes.c_char_p
        lib.qkn_last_error.argtypes = []
        lib.qkn_version.restype = ctypes.c_char_p
        lib.qkn_version.argtypes = []
        _lib = lib
        return lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        msg = load_library().qkn_last_error().decode(errors="replace")
        raise QKNormError(fn, status, msg)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return QKN_F32
    if t == torch.bfloat16:
        return QKN_BF16
    raise TypeError(f"unsupported dtype {t}; expected torch.float32 or torch.bfloat16")


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    return t


def _rows(t: torch.Tensor, name: str):
    _cuda(t, name)
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D with unit stride along the row")
    rows, cols = t.shape
    s0, s1 = t.stride()
    if cols > 1 and s1 != 1:
        raise ValueError(f"{name} must be 2-D with unit stride along the row")
    return rows, cols, max(s0, cols)


def _vec(t: torch.Tensor, name: str, n: int):
    _cuda(t, name)
    if t.dim() != 1 or t.shape[0] != n or (n > 1 and t.stride(0) != 1):
        raise ValueError(f"{name} must be a contiguous 1-D tensor of length {n}")


def _out2d(t: torch.Tensor, name: str, rows: int, cols: int, dtype: torch.dtype) -> torch.Tensor:
    """A caller-provided output: the exact shape and dtype, unit stride along the row."""
    _cuda(t, name)
    if t.dim() != 2 or tuple(t.shape) != (rows, cols) or t.dtype != dtype or (cols > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be a {dtype} [{rows}, {cols}] tensor with unit stride along the row")
    return t


def _device(ref: torch.Tensor, **tensors) -> torch.device:
    """Every CUDA tensor of a call lives on ref's device; the call is made there."""
    dev = ref.device
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device} but the call's inputs are on {dev}")
    return dev


class _On:
    """Makes the data's device current for the library call, only when it is not."""

    __slots__ = ("index", "prev")

    def __init__(self, dev: torch.device):
        self.index = dev.index

    def __enter__(self):
        self.prev = torch.cuda.current_device()
        if self.prev != self.index:
            torch.cuda.set_device(self.index)
        return self

    def __exit__(self, *exc):
        if self.prev != self.index:
            torch.cuda.set_device(self.prev)
        return False


# The current stream's raw handle without building a Stream object (the
# public route costs a few microseconds per call).
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> int:
    """Handle of `stream`, or of the current device's current stream."""
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def qknorm_fused(q: torch.Tensor, k: torch.Tensor | None, wq: torch.Tensor,
                 wk: torch.Tensor | None, eps: float = 1e-6, n_seg: int = 1, *,
                 q_out: torch.Tensor | None = None, k_out: torch.Tensor | None = None,
                 inplace: bool = False, stream=None):
    """QK-Norm of q [T, dq] and k [T, dk] (k may be None), one launch for both where
    their kernels agree (a row's result never depends on the other tensor).

    Returns ``(q_out, k_out)``.  With ``inplace=True`` the inputs are
    overwritten and returned; otherwise outputs are allocated unless given.
    Row pitches are taken from the tensors' strides (views of a fused QKV
    buffer work without copies).
    """
    T, dq, ldq = _rows(q, "q")
    act = _dtype_code(q.dtype)
    _vec(wq, "wq", dq)
    wdt = _dtype_code(wq.dtype)
    if k is not None:
        Tk, dk, ldk = _rows(k, "k")
        if Tk != T or k.dtype != q.dtype:
            raise ValueError("k must have q's row count and dtype")
        if wk is None:
            raise ValueError("wk is required with k")
        _vec(wk, "wk", dk)
        if wk.dtype != wq.dtype:
            raise ValueError("wk must have wq's dtype")
    else:
        dk, ldk = 0, 0
    if inplace:
        q_out_t, k_out_t = q, k
        q_ptr_out = k_ptr_out = None
        ldq_o, ldk_o = ldq, ldk
    else:
        q_out_t = q_out if q_out is not None else torch.empty((T, dq), dtype=q.dtype, device=q.device)
        _, _, ldq_o = _rows(_out2d(q_out_t, "q_out", T, dq, q.dtype), "q_out")
        q_ptr_out = q_out_t.data_ptr()
        if k is not None:
            k_out_t = k_out if k_out is not None else torch.empty((T, dk), dtype=k.dtype, device=k.device)
            _, _, ldk_o = _rows(_out2d(k_out_t, "k_out", T, dk, k.dtype), "k_out")
            k_ptr_out = k_out_t.data_ptr()
        else:
            k_out_t, k_ptr_out, ldk_o = None, None, 0
    dev = _device(q, k=k, wq=wq, wk=wk if k is not None else None, q_out=q_out_t, k_out=k_out_t)
    lib = load_library()
    with _On(dev):
        st = lib.qknorm_fused(q.data_ptr(), k.data_ptr() if k is not None else None,
                              wq.data_ptr(), wk.data_ptr() if k is not None else None,
                              q_ptr_out, k_ptr_out, T, dq, dk, ldq, ldk, ldq_o, ldk_o,
                              act, wdt, float(eps), int(n_seg), _stream(stream))
    _check("qknorm_fused", st)
    return q_out_t, k_out_t


HOST_WORKSPACE_BYTES = 3 * 64 * 1024 * 1024  # room for chunks up to 64 MiB


def qknorm_fused_host(q: torch.Tensor, k: torch.Tensor | None, wq: torch.Tensor,
                      wk: torch.Tensor | None, eps: float = 1e-6, n_seg: int = 1, *,
                      q_out: torch.Tensor | None = None, k_out: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None, stream=None):
    """QK-Norm of q [T, dq] and k [T, dk] held in HOST memory; results in host tensors.

    The rows stream through a device ``workspace`` (uint8 CUDA tensor,
    ``HOST_WORKSPACE_BYTES`` allocated when not given) in chunks whose upload,
    kernel and download overlap.  wq / wk live on the device.  Pinned host
    tensors let the copies run at link speed.  The call is asynchronous on
    ``stream``: synchronise it before reading the outputs.  Returns
    ``(q_out, k_out)``; ``q_out=q`` works in place.
    """
    def host_rows(t, name):
        if not isinstance(t, torch.Tensor) or t.is_cuda:
            raise ValueError(f"{name} must be a host (CPU) tensor")
        if t.dim() != 2 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 2-D tensor")
        return t.shape
    T, dq = host_rows(q, "q")
    act = _dtype_code(q.dtype)
    _vec(wq, "wq", dq)
    wdt = _dtype_code(wq.dtype)
    if k is not None:
        Tk, dk = host_rows(k, "k")
        if Tk != T or k.dtype != q.dtype:
            raise ValueError("k must have q's row count and dtype")
        if wk is None:
            raise ValueError("wk is required with k")
        _vec(wk, "wk", dk)
        if wk.dtype != wq.dtype:
            raise ValueError("wk must have wq's dtype")
    else:
        dk = 0
    pin = q.is_pinned()
    if q_out is None:
        q_out = torch.empty((T, dq), dtype=q.dtype, pin_memory=pin)
    if host_rows(q_out, "q_out") != (T, dq) or q_out.dtype != q.dtype:
        raise ValueError("q_out must match q")
    if k is not None:
        if k_out is None:
            k_out = torch.empty((T, dk), dtype=k.dtype, pin_memory=pin)
        if host_rows(k_out, "k_out") != (T, dk) or k_out.dtype != k.dtype:
            raise ValueError("k_out must match k")
    if workspace is None:
        workspace = torch.empty(HOST_WORKSPACE_BYTES, dtype=torch.uint8, device=wq.device)
    _cuda(workspace, "workspace")
    dev = _device(wq, wk=wk if k is not None else None, workspace=workspace)
    lib = load_library()
    with _On(dev):
        st = lib.qknorm_fused_host(q.data_ptr(), k.data_ptr() if k is not None else None,
                                   wq.data_ptr(), wk.data_ptr() if k is not None else None,
                                   q_out.data_ptr(), k_out.data_ptr() if k is not None else None,
                                   T, dq, dk, act, wdt, float(eps), int(n_seg),
                                   workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check("qknorm_fused_host", st)
    return q_out, (k_out if k is not None else None)


def rmsnorm_partial_stats(x: torch.Tensor, n_seg: int, *, out: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """Per-row sums of squares of n_seg contiguous segments: fp32 [rows, n_seg]."""
    rows, d, ld = _rows(x, "x")
    act = _dtype_code(x.dtype)
    if out is None:
        out = torch.empty((rows, n_seg), dtype=torch.float32, device=x.device)
    elif out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != (rows, n_seg):
        raise ValueError("out must be a contiguous fp32 tensor of shape [rows, n_seg]")
    dev = _device(x, out=_cuda(out, "out"))
    with _On(dev):
        st = load_library().rmsnorm_partial_stats(x.data_ptr(), rows, d, ld, act, int(n_seg),
                                                  out.data_ptr(), _stream(stream))
    _check("rmsnorm_partial_stats", st)
    return out


def flashnorm_fold_weights(w: torch.Tensor, W: torch.Tensor, *, k_major: bool = True,
                           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """FlashNorm fold W' = diag(w) W of W [K, N] (bf16); [N, K] when k_major else [K, N]."""
    _cuda(W, "W")
    if W.dim() != 2 or not W.is_contiguous() or W.dtype != torch.bfloat16:
        raise ValueError("W must be a contiguous bf16 [K, N] tensor")
    K, N = W.shape
    _vec(w, "w", K)
    shape = (N, K) if k_major else (K, N)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=W.device)
    elif tuple(out.shape) != shape or not out.is_contiguous() or out.dtype != torch.bfloat16:
        raise ValueError(f"out must be a contiguous bf16 tensor of shape {shape}")
    dev = _device(W, w=w, out=_cuda(out, "out"))
    with _On(dev):
        st = load_library().flashnorm_fold_weights(w.data_ptr(), W.data_ptr(), out.data_ptr(),
                                                   K, N, _dtype_code(w.dtype), int(bool(k_major)),
                                                   _stream(stream))
    _check("flashnorm_fold_weights", st)
    return out


def flashnorm_proj(x: torch.Tensor, W_folded: torch.Tensor, eps: float = 1e-6, *,
                   inv_rms: torch.Tensor | None = None, inv_rms_out: torch.Tensor | None = None,
                   out: torch.Tensor | None = None, k_major: bool = True, in_kernel_stats: bool = False,
                   stream=None) -> torch.Tensor:
    """y [M, N] = (x [M, K] @ W') * 1/rms(x), bf16 in/out, fp32 accumulate.

    W_folded is [N, K] (``k_major=True``, the layout the tensor cores read) or
    [K, N] (``k_major=False``: copied K-major inside the call first).  Without
    ``inv_rms`` the row statistics run as a separate pass overlapped with the
    projection, into ``inv_rms_out`` (allocated here when not given);
    ``in_kernel_stats=True`` computes them inside the projection kernel
    instead (no [M] workspace, slower).
    """
    _cuda(x, "x")
    _cuda(W_folded, "W_folded")
    if x.dim() != 2 or not x.is_contiguous() or x.dtype != torch.bfloat16:
        raise ValueError("x must be a contiguous bf16 [M, K] tensor")
    if W_folded.dim() != 2 or not W_folded.is_contiguous() or W_folded.dtype != torch.bfloat16:
        raise ValueError("W_folded must be a contiguous bf16 2-D tensor")
    M, K = x.shape
    N, K2 = W_folded.shape if k_major else (W_folded.shape[1], W_folded.shape[0])
    if K2 != K:
        raise ValueError(f"W_folded has K={K2} but x has K={K}")
    for name, t in (("inv_rms", inv_rms), ("inv_rms_out", inv_rms_out)):
        if t is not None:
            _vec(t, name, M)
            if t.dtype != torch.float32:
                raise ValueError(f"{name} must be fp32")
    if inv_rms is None and inv_rms_out is None and not in_kernel_stats:
        inv_rms_out = torch.empty(M, dtype=torch.float32, device=x.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif tuple(out.shape) != (M, N) or not out.is_contiguous() or out.dtype != torch.bfloat16:
        raise ValueError("out must be a contiguous bf16 [M, N] tensor")
    dev = _device(x, W_folded=W_folded, inv_rms=inv_rms, inv_rms_out=inv_rms_out, out=_cuda(out, "out"))
    with _On(dev):
        st = load_library().flashnorm_proj(
            x.data_ptr(), W_folded.data_ptr(), out.data_ptr(), M, N, K, 1 if k_major else 0, float(eps),
            inv_rms.data_ptr() if inv_rms is not None else None,
            inv_rms_out.data_ptr() if inv_rms_out is not None else None, _stream(stream))
    _check("flashnorm_proj", st)
    return out


def flashnorm_inv_rms(x: torch.Tensor, eps: float = 1e-6, *, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """FlashNorm's row statistic: fp32 [M] 1/rms of the rows of bf16 x [M, K]."""
    _cuda(x, "x")
    if x.dim() != 2 or not x.is_contiguous() or x.dtype != torch.bfloat16:
        raise ValueError("x must be a contiguous bf16 [M, K] tensor")
    M, K = x.shape
    if out is None:
        out = torch.empty(M, dtype=torch.float32, device=x.device)
    else:
        _vec(out, "out", M)
        if out.dtype != torch.float32:
            raise ValueError("out must be fp32")
    dev = _device(x, out=out)
    with _On(dev):
        st = load_library().flashnorm_inv_rms(x.data_ptr(), out.data_ptr(), M, K, float(eps), _stream(stream))
    _check("flashnorm_inv_rms", st)
    return out


def rmsnorm_apply_partials(x: torch.Tensor, w: torch.Tensor, partial: torch.Tensor, d_full: int,
                           eps: float = 1e-6, *, out: torch.Tensor | None = None,
                           inplace: bool = False, stream=None) -> torch.Tensor:
    """Normalise the shard x [rows, d] given every row's partial sums of squares.

    ``partial`` is fp32 and 2-D: [rows, n_part] (e.g. rmsnorm_partial_stats
    output) or [n_part, rows] (e.g. an all-gather of per-shard partials); the
    layout is read from its strides and its first dimension's length.
    ``d_full`` is the width of the whole row the partials cover.
    """
    rows, d, ld = _rows(x, "x")
    act = _dtype_code(x.dtype)
    _vec(w, "w", d)
    _cuda(partial, "partial")
    if partial.dtype != torch.float32 or partial.dim() != 2:
        raise ValueError("partial must be a 2-D fp32 tensor")
    if partial.shape[0] == rows:
        n_part, prs, ps = partial.shape[1], partial.stride(0), partial.stride(1)
    elif partial.shape[1] == rows:
        n_part, prs, ps = partial.shape[0], partial.stride(1), partial.stride(0)
    else:
        raise ValueError(f"partial {tuple(partial.shape)} does not match {rows} rows")
    if inplace:
        y, ldo = x, ld
    else:
        y = out if out is not None else torch.empty((rows, d), dtype=x.dtype, device=x.device)
        _, _, ldo = _rows(_out2d(y, "out", rows, d, x.dtype), "out")
    dev = _device(x, w=w, partial=partial, out=y)
    with _On(dev):
        st = load_library().rmsnorm_apply_partials(
            x.data_ptr(), w.data_ptr(), y.data_ptr(), rows, d, ld, ldo, partial.data_ptr(), int(n_part),
            int(prs), int(ps), int(d_full), act, _dtype_code(w.dtype), float(eps), _stream(stream))
    _check("rmsnorm_apply_partials", st)
    return y


def qkv_norm_proj(x: torch.Tensor, W_folded: torch.Tensor, nq: int, nk: int, nv: int,
                  wq: torch.Tensor, wk: torch.Tensor, wv: torch.Tensor | None, eps: float = 1e-6,
                  n_seg: int = 1, *, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """[q | k | v] = per-group RMSNorm of x W_folded^T; the pre-attention RMSNorm eliminated."""
    _cuda(x, "x")
    _cuda(W_folded, "W_folded")
    if x.dim() != 2 or not x.is_contiguous() or x.dtype != torch.bfloat16:
        raise ValueError("x must be a contiguous bf16 [M, K] tensor")
    M, K = x.shape
    N = nq + nk + nv
    if tuple(W_folded.shape) != (N, K) or not W_folded.is_contiguous() or W_folded.dtype != torch.bfloat16:
        raise ValueError(f"W_folded must be a contiguous bf16 [{N}, {K}] tensor")
    _vec(wq, "wq", nq)
    _vec(wk, "wk", nk)
    if nv > 0:
        _vec(wv, "wv", nv)
    for name, t in (("wk", wk), ("wv", wv if nv > 0 else None)):
        if t is not None and t.dtype != wq.dtype:
            raise ValueError(f"{name} must have wq's dtype")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif not out.is_contiguous():
        raise ValueError("out must be contiguous")
    _out2d(out, "out", M, N, torch.bfloat16)
    dev = _device(x, W_folded=W_folded, wq=wq, wk=wk, wv=wv if nv > 0 else None, out=out)
    with _On(dev):
        st = load_library().qkv_norm_proj(
            x.data_ptr(), W_folded.data_ptr(), out.data_ptr(), M, K, nq, nk, nv, wq.data_ptr(),
            wk.data_ptr(), wv.data_ptr() if (wv is not None and nv > 0) else None, _dtype_code(wq.dtype),
            float(eps), int(n_seg), _stream(stream))
    _check("qkv_norm_proj", st)
    return out


def qkv_proj_qknorm_workspace_bytes(M: int, nq: int, nk: int, nv: int) -> int:
    """Device scratch qkv_proj_qknorm needs for these sizes (bytes)."""
    return int(load_library().qkv_proj_qknorm_workspace_bytes(M, nq, nk, nv))


def qkv_proj_qknorm(x: torch.Tensor, W_folded: torch.Tensor, nq: int, nk: int, nv: int,
                    wq: torch.Tensor, wk: torch.Tensor, eps: float = 1e-6, eps_qk: float | None = None, *,
                    input_norm: bool = True, inv_rms: torch.Tensor | None = None,
                    inv_rms_out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """[q | k | v] = QK-Norm of RMSNorm(x) W in one GEMM (q, k normalised in the epilogue).

    The input norm's weights are folded into ``W_folded`` ([nq+nk+nv, K],
    from ``flashnorm_fold_weights``).  Its 1/rms comes from ``inv_rms`` when
    given, else a statistics pass writes it to ``inv_rms_out`` (allocated when
    ``input_norm`` and not given); ``input_norm=False`` uses x unscaled.
    ``eps_qk`` defaults to ``eps``.  ``workspace`` (uint8 CUDA tensor of at
    least ``qkv_proj_qknorm_workspace_bytes``) avoids an allocation inside
    the call.
    """
    _cuda(x, "x")
    _cuda(W_folded, "W_folded")
    if x.dim() != 2 or not x.is_contiguous() or x.dtype != torch.bfloat16:
        raise ValueError("x must be a contiguous bf16 [M, K] tensor")
    M, K = x.shape
    N = nq + nk + nv
    if tuple(W_folded.shape) != (N, K) or not W_folded.is_contiguous() or W_folded.dtype != torch.bfloat16:
        raise ValueError(f"W_folded must be a contiguous bf16 [{N}, {K}] tensor")
    _vec(wq, "wq", nq)
    _vec(wk, "wk", nk)
    if wk.dtype != wq.dtype:
        raise ValueError("wk must have wq's dtype")
    if inv_rms is not None:
        _vec(inv_rms, "inv_rms", M)
        if inv_rms.dtype != torch.float32:
            raise ValueError("inv_rms must be fp32")
    elif input_norm and inv_rms_out is None:
        inv_rms_out = torch.empty(M, dtype=torch.float32, device=x.device)
    if inv_rms_out is not None:
        _vec(inv_rms_out, "inv_rms_out", M)
        if inv_rms_out.dtype != torch.float32:
            raise ValueError("inv_rms_out must be fp32")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif not out.is_contiguous():
        raise ValueError("out must be contiguous")
    _out2d(out, "out", M, N, torch.bfloat16)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _cuda(workspace, "workspace")
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    dev = _device(x, W_folded=W_folded, wq=wq, wk=wk, inv_rms=inv_rms, inv_rms_out=inv_rms_out,
                  workspace=workspace, out=out)
    with _On(dev):
        st = load_library().qkv_proj_qknorm(
            x.data_ptr(), W_folded.data_ptr(), out.data_ptr(), M, K, nq, nk, nv,
            wq.data_ptr(), wk.data_ptr(), _dtype_code(wq.dtype), float(eps),
            float(eps if eps_qk is None else eps_qk),
            inv_rms.data_ptr() if inv_rms is not None else None,
            inv_rms_out.data_ptr() if (inv_rms is None and inv_rms_out is not None) else None,
            ws_ptr, ws_bytes, _stream(stream))
    _check("qkv_proj_qknorm", st)
    return out
