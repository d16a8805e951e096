"""Seeded synthetic inputs for the QK-Norm and FlashNorm workloads.

This module only draws random numbers: it holds none of the normalisation
arithmetic, so both the CUDA path's callers (tests, benchmark) and the oracle's
callers can share it without sharing any of the method.

Recipe (one ``torch.Generator`` seeded with ``seed`` on the requested device;
tensors are drawn in fp32 in the fixed order listed, then rounded once to the
activation dtype with round-to-nearest-even):

* ``q`` then ``k``: i.i.d. normal with the workload's standard deviation;
* ``wq`` then ``wk``: i.i.d. ``N(1, 0.1)`` (second argument = standard deviation),
  stored in the activation dtype;
* ``outliers`` workloads: then one seeded permutation per tensor (q first) whose
  first ``floor(0.01 * d)`` entries pick the outlier channels, scaled by 20
  before rounding;
* ``token_scale`` workloads: then one draw per token ``s = exp(U(ln 0.1, ln 10))``
  shared by that token's q row and k row, applied before rounding.

The values depend on the device the generator runs on (torch's CPU and CUDA
generators are different streams); every parity check therefore feeds the
oracle the exact values the GPU saw, copied back to the host.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = [
    "QKNormWorkload",
    "FlashNormWorkload",
    "QKNORM_WORKLOADS",
    "FLASHNORM_WORKLOAD",
    "make_qknorm_inputs",
    "make_flashnorm_inputs",
    "torch_dtype",
]


@dataclass(frozen=True)
class QKNormWorkload:
    name: str
    tokens: int
    dq: int
    dk: int
    dtype: str  # "f32" or "bf16": activations and weights
    n_seg: int
    eps: float
    x_std: float
    dist: str  # "normal" | "outliers" | "token_scale"
    description: str

    def algorithmic_bytes(self, tokens: int | None = None) -> int:
        """Bytes one pass must move: read q,k + write q,k + read both weights once."""
        t = self.tokens if tokens is None else tokens
        es = 4 if self.dtype == "f32" else 2
        return t * (self.dq + self.dk) * 2 * es + (self.dq + self.dk) * es


@dataclass(frozen=True)
class FlashNormWorkload:
    name: str
    M: int
    K: int
    N: int
    eps: float
    description: str

    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    def algorithmic_bytes(self) -> int:
        """x read + W' read + Y written (bf16), the GEMM's compulsory traffic."""
        return 2 * (self.M * self.K + self.K * self.N + self.M * self.N)


QKNORM_WORKLOADS = {
    w.name: w
    for w in [
        QKNormWorkload("tiny", 64, 4096, 4096, "f32", 1, 1e-6, 1.0, "normal",
                       "Tiny QK-Norm: 64 tokens, q/k dim 4096, fp32, n_seg=1"),
        QKNormWorkload("decode", 256, 5120, 5120, "bf16", 4, 1e-6, 1.0, "outliers",
                       "Decode-batch QK-Norm: 256 tokens, q/k dim 5120, bf16, 1% outlier "
                       "channels x20, n_seg=4"),
        QKNormWorkload("prefill_gqa", 16384, 5120, 1024, "bf16", 8, 1e-6, 1.0, "normal",
                       "Prefill GQA QK-Norm: 16384 tokens, q dim 5120 (40x128), k dim 1024 "
                       "(8x128), bf16, n_seg=8"),
        QKNormWorkload("long_context", 131072, 4096, 4096, "bf16", 8, 1e-6, 2.0, "token_scale",
                       "Long-context QK-Norm: 131072 tokens, q/k dim 4096, bf16, per-token "
                       "log-uniform scale in [0.1, 10], n_seg=8"),
        # not one of the stated configurations: rows narrow enough to be held in
        # registers (a small model's q and k, 8 heads x 128), measured beside them
        QKNormWorkload("narrow_rows", 131072, 1024, 1024, "bf16", 4, 1e-6, 1.0, "normal",
                       "Narrow-row QK-Norm: 131072 tokens, q/k dim 1024 (8x128), bf16, n_seg=4"),
    ]
}

FLASHNORM_WORKLOAD = FlashNormWorkload(
    "flashnorm_proj", 8192, 4096, 12288, 1e-6,
    "FlashNorm norm-then-project: x[8192,4096] bf16, w folded into W[4096,12288] bf16, "
    "1/rms applied in the GEMM epilogue")


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_qknorm_inputs(wl: QKNormWorkload | str, seed: int = 0, device="cpu",
                       tokens: int | None = None, dq: int | None = None,
                       dk: int | None = None) -> dict:
    """Draw q [T,dq], k [T,dk], wq [dq], wk [dk] for a QK-Norm workload.

    ``tokens``/``dq``/``dk`` override the workload's sizes while keeping its
    distribution (used for oracle-sized parity cases).  Returns contiguous
    tensors on ``device`` in the workload's dtype.
    """
    if isinstance(wl, str):
        wl = QKNORM_WORKLOADS[wl]
    T = wl.tokens if tokens is None else tokens
    dq = wl.dq if dq is None else dq
    dk = wl.dk if dk is None else dk
    g = _gen(seed, device)
    f32 = torch.float32
    q = torch.randn(T, dq, generator=g, device=device, dtype=f32) * wl.x_std
    k = torch.randn(T, dk, generator=g, device=device, dtype=f32) * wl.x_std
    wq = 1.0 + 0.1 * torch.randn(dq, generator=g, device=device, dtype=f32)
    wk = 1.0 + 0.1 * torch.randn(dk, generator=g, device=device, dtype=f32)
    if wl.dist == "outliers":
        for x in (q, k):
            d = x.shape[1]
            n_out = int(math.floor(0.01 * d))
            chans = torch.randperm(d, generator=g, device=device)[:n_out]
            x[:, chans] *= 20.0
    elif wl.dist == "token_scale":
        u = torch.rand(T, generator=g, device=device, dtype=f32)
        lo, hi = math.log(0.1), math.log(10.0)
        s = torch.exp(lo + (hi - lo) * u)
        q *= s[:, None]
        k *= s[:, None]
    dt = torch_dtype(wl.dtype)
    return {
        "q": q.to(dt).contiguous(),
        "k": k.to(dt).contiguous(),
        "wq": wq.to(dt).contiguous(),
        "wk": wk.to(dt).contiguous(),
        "n_seg": wl.n_seg,
        "eps": wl.eps,
    }


def make_flashnorm_inputs(seed: int = 0, device="cpu", M: int | None = None,
                          K: int | None = None, N: int | None = None) -> dict:
    """Draw x [M,K] ~ N(0,1), w [K] ~ N(1,0.1), W [K,N] ~ N(0, 1/sqrt(K)) in bf16.

    Drawn in that order from one generator, in fp32, then rounded to bf16.
    """
    wl = FLASHNORM_WORKLOAD
    M = wl.M if M is None else M
    K = wl.K if K is None else K
    N = wl.N if N is None else N
    g = _gen(seed, device)
    f32 = torch.float32
    x = torch.randn(M, K, generator=g, device=device, dtype=f32)
    w = 1.0 + 0.1 * torch.randn(K, generator=g, device=device, dtype=f32)
    W = torch.randn(K, N, generator=g, device=device, dtype=f32) * (1.0 / math.sqrt(K))
    bf = torch.bfloat16
    return {"x": x.to(bf).contiguous(), "w": w.to(bf).contiguous(),
            "W": W.to(bf).contiguous(), "eps": wl.eps}


def make_qkv_norm_weights(nq: int, nk: int, seed: int = 0, device="cpu"):
    """QK-Norm weights for the QKV projection workload: wq [nq], wk [nk] ~ N(1, 0.1) in bf16.

    Drawn in that order from one generator, in fp32, then rounded to bf16.
    """
    g = _gen(seed + 1, device)
    f32 = torch.float32
    wq = 1.0 + 0.1 * torch.randn(nq, generator=g, device=device, dtype=f32)
    wk = 1.0 + 0.1 * torch.randn(nk, generator=g, device=device, dtype=f32)
    return wq.to(torch.bfloat16).contiguous(), wk.to(torch.bfloat16).contiguous()
