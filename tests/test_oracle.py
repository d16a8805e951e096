"""Pins for the fp64 oracle (CPU only).

The pages print no worked example with numbers, so every pin here is a closed
form, an invariant or a brute-force / library special case fixed by the
mathematics of RMSNorm (SwiftQK, abstract: QK-Norm is an RMSNorm over the full
vector, built from scalar partial sums) and of FlashNorm (abstract, items (i)
and (ii): fold w into the next weight, defer 1/rms to the matmul output).
Each test names the mistake it is there to catch.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(1234)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(*shape):
    return RNG.standard_normal(shape)


# ----------------------------------------------------------------------------- RMSNorm


@pytest.mark.parametrize("d", [1, 2, 7, 64, 1000, 4096])
def test_unit_rms_when_weights_one_and_eps_zero(d):
    # catches: sum instead of mean, missing sqrt, eps added to the wrong place
    x = rand(5, d) * 3.0
    y = oracle.rmsnorm(x, np.ones(d), 0.0)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-13)


@pytest.mark.parametrize("c", [1e-3, 7.0, 1e3, -2.5])
def test_scale_invariance(c):
    # RMSNorm(c x) = sign(c) RMSNorm(x) when eps = 0
    x, w = rand(4, 96), rand(96)
    a = oracle.rmsnorm(c * x, w, 0.0)
    b = oracle.rmsnorm(x, w, 0.0)
    np.testing.assert_allclose(a, math.copysign(1.0, c) * b, rtol=1e-13, atol=1e-300)


def test_eps_breaks_scale_invariance_in_the_right_direction():
    # eps is added to mean(x^2): a tiny input is shrunk, a large one is not.
    x, w = rand(3, 32), np.ones(32)
    small = oracle.rmsnorm(1e-6 * x, w, 1e-6)
    big = oracle.rmsnorm(1e3 * x, w, 1e-6)
    assert np.all((small ** 2).mean(axis=1) < 1e-3)
    np.testing.assert_allclose((big ** 2).mean(axis=1), 1.0, rtol=1e-10)


def test_pm_one_row_gives_x_times_w():
    # rms of a +-1 vector is exactly 1, so y = x * w exactly (eps = 0)
    d = 257
    x = np.where(RNG.random((3, d)) < 0.5, -1.0, 1.0)
    w = rand(d)
    np.testing.assert_array_equal(oracle.rmsnorm(x, w, 0.0), x * w)


@pytest.mark.parametrize("c", [3.0, -0.125])
def test_one_hot(c):
    # x = c e_i: mean(x^2) = c^2/d, so y_i = sign(c) sqrt(d) w_i and 0 elsewhere.
    # catches: sum instead of mean (factor sqrt(d)), wrong weight index
    d, i = 64, 37
    x = np.zeros((1, d))
    x[0, i] = c
    w = 1.0 + np.arange(d) / 10.0
    y = oracle.rmsnorm(x, w, 0.0)
    expect = np.zeros((1, d))
    expect[0, i] = math.copysign(1.0, c) * math.sqrt(d) * w[i]
    np.testing.assert_allclose(y, expect, rtol=1e-14, atol=0)


def test_constant_row():
    # x = c * 1 -> y = sign(c) * w
    d = 100
    w = rand(d)
    for c in (0.3, -12.0):
        y = oracle.rmsnorm(np.full((1, d), c), w, 0.0)
        np.testing.assert_allclose(y[0], math.copysign(1.0, c) * w, rtol=1e-14)


def test_d_equals_one():
    # a single element: y = sign(x) * w
    x = np.array([[2.5], [-0.01], [7e10]])
    y = oracle.rmsnorm(x, np.array([0.75]), 0.0)
    np.testing.assert_allclose(y[:, 0], [0.75, -0.75, 0.75], rtol=1e-15)


def test_zero_row():
    # eps > 0: 0 / sqrt(eps) = 0; eps = 0: 0/0 = NaN (IEEE)
    x = np.zeros((1, 16))
    w = np.ones(16)
    assert np.all(oracle.rmsnorm(x, w, 1e-6) == 0.0)
    assert np.all(np.isnan(oracle.rmsnorm(x, w, 0.0)))


def test_permutation_equivariance():
    # permuting channels of x and w together permutes y: catches a weight
    # indexed by row or a shifted weight index
    x, w = rand(6, 50), rand(50)
    p = RNG.permutation(50)
    np.testing.assert_allclose(oracle.rmsnorm(x[:, p], w[p], 1e-3),
                               oracle.rmsnorm(x, w, 1e-3)[:, p], rtol=1e-14)


def test_rows_are_independent():
    # each row's statistic uses only that row (catches a whole-matrix mean)
    x, w = rand(4, 24), rand(24)
    full = oracle.rmsnorm(x, w, 1e-4)
    for r in range(4):
        np.testing.assert_array_equal(oracle.rmsnorm(x[r:r + 1], w, 1e-4)[0], full[r])


def test_golden_closed_forms():
    # hand-derived values, see tests/golden/rmsnorm_closed_forms.json
    with open(os.path.join(GOLDEN, "rmsnorm_closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 3
    for c in cases:
        y = oracle.rmsnorm(np.array([c["x"]]), np.array(c["w"]), c["eps"])
        expect = [eval(e, {"sqrt": math.sqrt}) for e in c["y"]]  # noqa: S307 (fixture exprs)
        np.testing.assert_allclose(y[0], expect, rtol=1e-15, err_msg=c["name"])


# ------------------------------------------------------------------ partial sums / combine


@pytest.mark.parametrize("n_seg", [1, 2, 4, 8])
def test_partials_sum_to_full_statistic(n_seg):
    x = rand(7, 640)
    p = oracle.segment_partials(x, n_seg)
    full = oracle.segment_partials(x, 1)[:, 0]
    np.testing.assert_allclose(p.sum(axis=1), full, rtol=1e-13)
    np.testing.assert_allclose(oracle.combine_partials(p), full, rtol=1e-13)


def test_partials_are_contiguous_segments():
    # segments are contiguous slices, not interleaved: row = [1]*L + [2]*L + [3]*L
    L = 5
    x = np.concatenate([np.full(L, 1.0), np.full(L, 2.0), np.full(L, 3.0)])[None, :]
    np.testing.assert_array_equal(oracle.segment_partials(x, 3), [[L * 1.0, L * 4.0, L * 9.0]])


def test_partials_closed_forms():
    d = 64
    pm = np.where(RNG.random((2, d)) < 0.5, -1.0, 1.0)
    np.testing.assert_array_equal(oracle.segment_partials(pm, 8), np.full((2, 8), d / 8))
    one_hot = np.zeros((1, d))
    one_hot[0, 20] = -3.0  # segment 20 // 8 = 2
    expect = np.zeros((1, 8))
    expect[0, 2] = 9.0
    np.testing.assert_array_equal(oracle.segment_partials(one_hot, 8), expect)
    x = rand(3, d)
    np.testing.assert_array_equal(oracle.segment_partials(x, d), x * x)


def test_partials_reject_ragged_split():
    with pytest.raises(ValueError):
        oracle.segment_partials(rand(2, 10), 3)


def test_combine_is_left_to_right():
    # ((1e16 + 1) - 1e16) = 0 in fp64, any other order of these three gives 1 or 0
    # differently; pins the fixed left-to-right combine order
    p = np.array([[1e16, 1.0, -1e16], [1.0, 1e16, -1e16], [1.0, 2.0, 3.0]])
    np.testing.assert_array_equal(oracle.combine_partials(p), [0.0, 0.0, 6.0])
    p2 = np.array([[1e16, -1e16, 1.0]])
    np.testing.assert_array_equal(oracle.combine_partials(p2), [1.0])


def test_inv_rms_closed_form_and_consistency():
    x = np.array([[3.0, 4.0], [1.0, 1.0]])
    np.testing.assert_allclose(oracle.inv_rms(x, 0.0), [1 / math.sqrt(12.5), 1.0], rtol=1e-15)
    np.testing.assert_allclose(oracle.inv_rms(x, 0.5), [1 / math.sqrt(13.0), 1 / math.sqrt(1.5)],
                               rtol=1e-15)
    xr = rand(5, 33)
    np.testing.assert_allclose(oracle.rmsnorm(xr, np.ones(33), 1e-2),
                               xr * oracle.inv_rms(xr, 1e-2)[:, None], rtol=1e-14)


# ------------------------------------------------------------------------------ FlashNorm


def _brute_matmul(a, b):
    # textbook triple loop, pure Python, tiny shapes only
    M, K = a.shape
    K2, N = b.shape
    assert K == K2
    out = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            s = 0.0
            for k in range(K):
                s += a[m, k] * b[k, n]
            out[m, n] = s
    return out


@pytest.mark.parametrize("M,K,N", [(1, 1, 1), (3, 5, 2), (8, 8, 8), (2, 7, 5)])
def test_flashnorm_identity_brute_force(M, K, N):
    # FlashNorm (ii): (x diag(w) W) / rms(x) == RMSNorm(x) W, exact in real arithmetic
    x, w, W = rand(M, K), rand(K), rand(K, N)
    eps = 1e-3
    ref = _brute_matmul(oracle.rmsnorm(x, w, eps), W)
    np.testing.assert_allclose(oracle.norm_then_project(x, w, W, eps), ref, rtol=1e-12, atol=1e-14)
    folded = oracle.flashnorm_deferred(x, oracle.fold_weights(w, W), eps)
    np.testing.assert_allclose(folded, ref, rtol=1e-12, atol=1e-14)


def test_norm_then_project_matches_library_matmul():
    # special case that reduces to a library routine: numpy's matmul
    x, w, W = rand(16, 48), rand(48), rand(48, 24)
    np.testing.assert_allclose(oracle.norm_then_project(x, w, W, 1e-6),
                               oracle.rmsnorm(x, w, 1e-6) @ W, rtol=1e-11, atol=1e-13)


def test_fold_weights():
    # FlashNorm (i): w = 1 leaves W unchanged; row k of W is scaled by w[k] (not column)
    W = rand(6, 4)
    np.testing.assert_array_equal(oracle.fold_weights(np.ones(6), W), W)
    w = np.array([2.0, -1.0, 0.5, 0.0, 4.0, 1.0])
    np.testing.assert_array_equal(oracle.fold_weights(w, W), W * w[:, None])
    Wn = rand(3, 5)  # non-square: catches a transposed scale
    np.testing.assert_array_equal(oracle.fold_weights(np.array([1.0, 2.0, 3.0]), Wn)[2], 3.0 * Wn[2])


def test_deferred_with_unit_weights_and_identity_projection():
    # W' = I: (x I)/rms(x) is RMSNorm(x) with w = 1
    x = rand(4, 9)
    np.testing.assert_allclose(oracle.flashnorm_deferred(x, np.eye(9), 0.0),
                               oracle.rmsnorm(x, np.ones(9), 0.0), rtol=1e-14)


# ------------------------------------------------------------------------- bf16 rounding


def test_round_bf16_matches_torch_on_float32_values():
    # for values that are already binary32 there is no double-rounding issue,
    # so torch's float32 -> bf16 (RNE) is a library pin
    v = np.concatenate([
        RNG.standard_normal(20000).astype(np.float32),
        (RNG.standard_normal(5000) * 1e30).astype(np.float32),
        (RNG.standard_normal(5000) * 1e-38).astype(np.float32),  # subnormal range
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38], dtype=np.float32),
    ])
    expect = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.round_bf16_bits(v.astype(np.float64)), expect)


def test_round_bf16_ties_and_double_rounding():
    u = 2.0 ** -7  # bf16 ulp at 1
    cases = {
        1.0 + u / 2: 0x3F80,                 # tie -> even (1.0)
        1.0 + 3 * u / 2: 0x3F82,             # tie -> even (1 + 2u)
        1.0 + u / 2 + 2.0 ** -40: 0x3F81,    # just above the tie: up (float32 first would tie down)
        -(1.0 + u / 2 + 2.0 ** -40): 0xBF81,
        1.0 + u / 2 - 2.0 ** -40: 0x3F80,
        (2.0 - 2.0 ** -8) * 2.0 ** 127: 0x7F80,   # halfway to 2^128: overflows to inf
        (2.0 - 2.0 ** -7) * 2.0 ** 127: 0x7F7F,   # max finite
        2.0 ** -133: 0x0001,                       # smallest subnormal
        2.0 ** -134: 0x0000,                       # tie between 0 and 2^-133 -> even (0)
        -0.0: 0x8000,
        math.inf: 0x7F80,
        -math.inf: 0xFF80,
    }
    v = np.array(list(cases.keys()))
    np.testing.assert_array_equal(oracle.round_bf16_bits(v), np.array(list(cases.values()), np.uint16))
    nan = oracle.round_bf16_bits(np.array([math.nan]))[0]
    assert (nan & 0x7FFF) > 0x7F80


def test_oracle_threads_positive():
    assert oracle.threads() >= 1


# --------------------------------------------------------------- RMSNorm elimination


@pytest.mark.parametrize("eps_post", [0.0, 1e-6])
def test_rmsnorm_elimination_identity(eps_post):
    # FlashNorm (abstract): RMSNorm -> linear -> RMSNorm lets the first RMSNorm go.
    # With the first norm's eps = 0, RMSNorm(RMSNorm(x; w) W; v) = RMSNorm((x diag(w)) W; v)
    # because the first norm only scales each row of the product by 1/rms(x) > 0.
    x, w, W, v = rand(6, 40), rand(40), rand(40, 24), rand(24)
    full = oracle.rmsnorm(oracle.norm_then_project(x, w, W, 0.0), v, eps_post)
    eliminated = oracle.rmsnorm(x @ oracle.fold_weights(w, W), v, eps_post)  # numpy matmul: a library step
    tol = 1e-12 if eps_post == 0.0 else 1e-6
    np.testing.assert_allclose(eliminated, full, rtol=tol, atol=1e-12)


def test_rmsnorm_elimination_needs_the_second_norm():
    # without the second norm the row scale 1/rms(x) survives: catches an identity applied too widely
    x, w, W = rand(4, 16) * 5, rand(16), rand(16, 8)
    assert not np.allclose(oracle.norm_then_project(x, w, W, 0.0), x @ oracle.fold_weights(w, W))


# --------------------------------------------------------------- QKV projection + QK-Norm


def _brute_qkv(x, w_in, W, wq, wk, nq, nk, eps, eps_qk):
    # written out element by element in pure Python: the definition, nothing shared
    M, K = len(x), len(x[0])
    N = len(W[0])
    out = [[0.0] * N for _ in range(M)]
    for m in range(M):
        r = 1.0 / math.sqrt(sum(v * v for v in x[m]) / K + eps)
        u = [sum(x[m][k] * r * w_in[k] * W[k][n] for k in range(K)) for n in range(N)]
        for lo, hi, w in ((0, nq, wq), (nq, nq + nk, wk)):
            s = sum(u[n] * u[n] for n in range(lo, hi))
            inv = 1.0 / math.sqrt(s / (hi - lo) + eps_qk)
            for n in range(lo, hi):
                out[m][n] = u[n] * inv * w[n - lo]
        for n in range(nq + nk, N):
            out[m][n] = u[n]
    return np.array(out)


@pytest.mark.parametrize("eps,eps_qk", [(0.0, 0.0), (1e-6, 1e-6), (0.3, 0.05)])
def test_qkv_qknorm_brute_force(eps, eps_qk):
    x, w_in, W = rand(3, 5), rand(5), rand(5, 11)
    wq, wk = rand(4), rand(3)
    got = oracle.qkv_proj_qknorm(x, w_in, W, wq, wk, 4, 3, eps, eps_qk)
    ref = _brute_qkv(x.tolist(), w_in.tolist(), W.tolist(), wq.tolist(), wk.tolist(), 4, 3, eps, eps_qk)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_qkv_qknorm_identity_projection_reduces_to_rmsnorm():
    # W = I, w_in = 1, eps = eps_qk = 0: the input norm only scales each row by a positive
    # factor, which QK-Norm removes, so q and k are plain RMSNorms of x's own slices and v
    # is the slice of RMSNorm(x)
    nq, nk, nv = 6, 4, 5
    d = nq + nk + nv
    x, wq, wk = rand(7, d), rand(nq), rand(nk)
    y = oracle.qkv_proj_qknorm(x, np.ones(d), np.eye(d), wq, wk, nq, nk, 0.0, 0.0)
    np.testing.assert_allclose(y[:, :nq], oracle.rmsnorm(x[:, :nq].copy(), wq, 0.0), rtol=1e-12)
    np.testing.assert_allclose(y[:, nq:nq + nk], oracle.rmsnorm(x[:, nq:nq + nk].copy(), wk, 0.0), rtol=1e-12)
    np.testing.assert_allclose(y[:, nq + nk:], oracle.rmsnorm(x, np.ones(d), 0.0)[:, nq + nk:], rtol=1e-12)


def test_qkv_qknorm_unit_rms_and_section_swap():
    x, w_in, W = rand(5, 16), rand(16), rand(16, 20)
    nq, nk = 8, 6
    y = oracle.qkv_proj_qknorm(x, w_in, W, np.ones(nq), np.ones(nk), nq, nk, 1e-6, 0.0)
    np.testing.assert_allclose(np.sqrt((y[:, :nq] ** 2).mean(1)), 1.0, rtol=1e-12)
    np.testing.assert_allclose(np.sqrt((y[:, nq:nq + nk] ** 2).mean(1)), 1.0, rtol=1e-12)
    # moving k's columns in front of q's (with their weights) moves the outputs the same way
    wq, wk = rand(nq), rand(nk)
    a = oracle.qkv_proj_qknorm(x, w_in, W, wq, wk, nq, nk, 1e-6, 1e-3)
    perm = np.r_[nq:nq + nk, 0:nq, nq + nk:20]
    b = oracle.qkv_proj_qknorm(x, w_in, W[:, perm], wk, wq, nk, nq, 1e-6, 1e-3)
    np.testing.assert_allclose(b, a[:, perm], rtol=1e-12, atol=1e-14)


def test_qkv_qknorm_without_input_norm_is_scale_free_on_q_and_k():
    # input_norm=False uses x as it is; q and k are still normalised, so scaling x changes only v
    x, W = rand(4, 12), rand(12, 14)
    a = oracle.qkv_proj_qknorm(x, None, W, np.ones(6), np.ones(4), 6, 4, 0.0, 0.0, input_norm=False)
    b = oracle.qkv_proj_qknorm(3 * x, None, W, np.ones(6), np.ones(4), 6, 4, 0.0, 0.0, input_norm=False)
    np.testing.assert_allclose(b[:, :10], a[:, :10], rtol=1e-12)
    np.testing.assert_allclose(b[:, 10:], 3 * a[:, 10:], rtol=1e-12)
