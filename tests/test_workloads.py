"""The seeded input generators: shapes, dtypes, seeding and the stated distributions."""
import math

import torch

from rmsnorm_qknorm_b200 import workloads as W


def test_shapes_and_dtypes_small_override():
    for name, wl in W.QKNORM_WORKLOADS.items():
        inp = W.make_qknorm_inputs(name, tokens=8)
        assert inp["q"].shape == (8, wl.dq) and inp["k"].shape == (8, wl.dk)
        assert inp["wq"].shape == (wl.dq,) and inp["wk"].shape == (wl.dk,)
        dt = W.torch_dtype(wl.dtype)
        assert all(inp[t].dtype == dt for t in ("q", "k", "wq", "wk"))
        assert inp["n_seg"] == wl.n_seg and inp["eps"] == wl.eps
        assert wl.dq % wl.n_seg == 0 and wl.dk % wl.n_seg == 0


def test_seeded_and_reproducible():
    a = W.make_qknorm_inputs("decode", tokens=4, seed=3)
    b = W.make_qknorm_inputs("decode", tokens=4, seed=3)
    c = W.make_qknorm_inputs("decode", tokens=4, seed=4)
    assert torch.equal(a["q"], b["q"]) and not torch.equal(a["q"], c["q"])


def test_weight_distribution():
    inp = W.make_qknorm_inputs("prefill_gqa", tokens=2)
    wq = inp["wq"].float()
    assert abs(wq.mean().item() - 1.0) < 0.01 and abs(wq.std().item() - 0.1) < 0.01


def test_outlier_channels():
    inp = W.make_qknorm_inputs("decode", tokens=512)
    q = inp["q"].float()
    col_std = q.std(dim=0)
    n_out = int((col_std > 10).sum())
    assert n_out == math.floor(0.01 * 5120)  # 51 channels scaled x20
    assert abs(col_std[col_std < 10].mean().item() - 1.0) < 0.05


def test_token_scale_range():
    inp = W.make_qknorm_inputs("long_context", tokens=2048, dq=256, dk=256)
    q, k = inp["q"].float(), inp["k"].float()
    rq = q.pow(2).mean(dim=1).sqrt()
    rk = k.pow(2).mean(dim=1).sqrt()
    # std 2 times a per-token scale in [0.1, 10], shared by q and k
    assert rq.min().item() > 0.1 * 2 * 0.7 and rq.max().item() < 10 * 2 * 1.3
    ratio = (rq / rk)
    assert 0.7 < ratio.median().item() < 1.3
    assert (rq.log().std().item()) > 1.0  # log-uniform over two decades


def test_flashnorm_inputs():
    inp = W.make_flashnorm_inputs(M=64, K=256, N=128)
    assert inp["x"].shape == (64, 256) and inp["W"].shape == (256, 128)
    assert inp["w"].shape == (256,)
    assert abs(inp["W"].float().std().item() - 1 / 16) < 0.005
    wl = W.FLASHNORM_WORKLOAD
    assert wl.flops() == 2 * 8192 * 4096 * 12288
