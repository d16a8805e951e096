"""Comparison rules shared by the parity tests (test-side only).

* fp32 outputs: per-element relative error |g - o| / |o| <= 1e-5 against the
  fp64 oracle; where the oracle is exactly 0 the output must be 0 too (the
  output is a product x * inv * w, so it has no cancellation).
* bf16 outputs: the output's bit pattern is within one bf16 ulp of the oracle
  value rounded once to bf16 (round-to-nearest-even), i.e. the sign-magnitude
  patterns differ by at most 1 step; +0 and -0 count as equal.
* fp32 partial sums: relative error <= 1e-5 against the fp64 partials.
* bf16 projection: relative Frobenius error <= 1e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

F32_REL_TOL = 1e-5
PARTIAL_REL_TOL = 1e-5
BF16_ULP_TOL = 1
PROJ_FROB_TOL = 1e-2


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_ulp_distance(g_bits: np.ndarray, o_bits: np.ndarray) -> np.ndarray:
    """Steps between two bf16 patterns on the ordered line (+0 == -0)."""
    return np.abs(_ordered(g_bits) - _ordered(o_bits))


def assert_bf16_close(gpu: torch.Tensor, ref64: np.ndarray, what: str = "") -> int:
    """GPU bf16 output vs fp64 oracle: within 1 ulp of RNE(oracle). Returns max ulp."""
    g = bf16_bits(gpu).reshape(ref64.shape)
    o = oracle.round_bf16_bits(ref64)
    g_nan = (g & 0x7FFF) > 0x7F80
    o_nan = (o & 0x7FFF) > 0x7F80
    assert np.array_equal(g_nan, o_nan), f"{what}: NaN pattern differs"
    dist = bf16_ulp_distance(g[~g_nan], o[~o_nan])
    worst = int(dist.max()) if dist.size else 0
    if worst > BF16_ULP_TOL:
        idx = np.unravel_index(np.argmax(bf16_ulp_distance(g, o) * (~g_nan)), g.shape)
        raise AssertionError(
            f"{what}: {int((dist > BF16_ULP_TOL).sum())} elements beyond {BF16_ULP_TOL} bf16 ulp; "
            f"worst {worst} ulp at {idx}: gpu bits {g[idx]:#06x} oracle {ref64[idx]!r} "
            f"(rounded {o[idx]:#06x})")
    return worst


def assert_f32_close(gpu: torch.Tensor, ref64: np.ndarray, tol: float = F32_REL_TOL,
                     what: str = "") -> float:
    """GPU fp32 output vs fp64 oracle: max relative error <= tol; exact zeros match."""
    g = gpu.detach().cpu().double().numpy().reshape(ref64.shape)
    zero = ref64 == 0
    assert np.all(g[zero] == 0), f"{what}: oracle zero but output nonzero"
    nz = ~zero
    rel = np.abs(g[nz] - ref64[nz]) / np.abs(ref64[nz])
    worst = float(rel.max()) if rel.size else 0.0
    assert np.all(np.isfinite(g[nz])), f"{what}: non-finite output where oracle is finite"
    assert worst <= tol, f"{what}: max relative error {worst:.3e} > {tol:.1e}"
    return worst


def frobenius_rel(gpu: torch.Tensor, ref64: np.ndarray) -> float:
    g = gpu.detach().cpu().double().numpy().reshape(ref64.shape)
    return float(np.linalg.norm(g - ref64) / np.linalg.norm(ref64))
