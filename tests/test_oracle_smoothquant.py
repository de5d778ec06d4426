"""Pins of the oracle's SmoothQuant smoothing ("27届大模型面试准备（十九）…" sec. 4.2):
closed forms of the migration factor, the page's reading of alpha = 0 and 1,
the exactness of the rewrite Y = (X diag(s)^-1)(diag(s) W), and the page's
claim that smoothing makes W8A8 on outlier activations more accurate."""
import math

import numpy as np
import pytest

import oracle
from workloads import make_activation, make_weight


def test_channel_absmax_hand_matrix():
    A = np.array([[1.0, -3.0, 0.5, 0.0],
                  [-2.0, 2.0, -0.25, 0.0],
                  [1.5, -1.0, 0.75, -0.0]], np.float32)
    out, st = oracle.channel_absmax(A)
    assert st == oracle.OK
    assert out.tolist() == [2.0, 3.0, 0.75, 0.0]


def test_channel_absmax_skips_and_reports_non_finite():
    A = np.array([[1.0, np.nan], [-4.0, 2.0]], np.float32)
    out, st = oracle.channel_absmax(A)
    assert st == oracle.ERR_NONFINITE
    assert out.tolist() == [4.0, 2.0]


@pytest.mark.parametrize("a,w,alpha,expect", [
    (4.0, 1.0, 0.5, 2.0), (1.0, 4.0, 0.5, 0.5), (9.0, 1.0, 0.5, 3.0),
    (5.0, 4.0, 0.0, 0.25),          # alpha = 0: 1 / max|W_j|
    (5.0, 7.0, 1.0, 5.0),           # alpha = 1: max|X_j|
    (8.0, 2.0, 0.25, 8.0 ** 0.25 / 2.0 ** 0.75),
])
def test_smooth_scale_closed_forms(a, w, alpha, expect):
    s, st = oracle.smooth_scales(np.array([a], np.float32), np.array([w], np.float32), alpha)
    assert st == oracle.OK
    assert s[0] == np.float32(expect)


def test_smooth_scale_clamps():
    # a weight statistic below 1e-5 is raised to 1e-5; s itself is at least 1e-5
    s, st = oracle.smooth_scales(np.array([9.0, 0.0], np.float32),
                                 np.array([0.0, 3.0], np.float32), 0.5)
    assert st == oracle.OK
    assert s[0] == np.float32(3.0 / math.sqrt(float(np.float32(1e-5))))
    assert s[1] == np.float32(1e-5)
    _, st = oracle.smooth_scales(np.ones(2, np.float32), np.ones(2, np.float32), 1.5)
    assert st == oracle.ERR_ARG


def test_alpha_extremes_flatten_one_side():
    """alpha = 1 moves everything to the weight: every column of X diag(s)^-1
    has max |.| = 1; alpha = 0 leaves it with the activations: every column of
    W diag(s) (clamp aside) has max |.| = 1.  An exponent swap fails both."""
    X = make_activation(32, 256, seed=3, outlier_dims=6).float().numpy()
    W = make_weight(64, 256, 0.02, seed=3).float().numpy()
    a, _ = oracle.channel_absmax(X)
    w, _ = oracle.channel_absmax(W)
    s1, _ = oracle.smooth_scales(a, w, 1.0)
    np.testing.assert_allclose(np.abs(X / s1).max(axis=0), 1.0, rtol=1e-6)
    s0, _ = oracle.smooth_scales(a, w, 0.0)
    np.testing.assert_allclose(np.abs(W * s0).max(axis=0), 1.0, rtol=1e-6)


def test_unit_scales_reduce_to_the_plain_quantizers():
    X = make_activation(8, 512, seed=5, outlier_dims=6)
    W = make_weight(16, 512, 0.02, seed=5)
    ones = np.ones(512, np.float32)
    q1, s1, _ = oracle.quant_act_i8_smoothed(X.float().numpy(), ones)
    q0, s0, _ = oracle.quant_act_i8(X.float().numpy())
    assert np.array_equal(q1, q0) and np.array_equal(s1, s0)
    q1, s1, _ = oracle.quantize_int8_rows_smoothed(W.float().numpy(), ones)
    q0, s0, _ = oracle.quantize_int8_rows(W.float().numpy())
    assert np.array_equal(q1, q0) and np.array_equal(s1, s0)


def _w8a8(X, W, s=None):
    if s is None:
        qx, sx, _ = oracle.quant_act_i8(X)
        qw, sw, _ = oracle.quantize_int8_rows(W)
    else:
        qx, sx, _ = oracle.quant_act_i8_smoothed(X, s)
        qw, sw, _ = oracle.quantize_int8_rows_smoothed(W, s)
    return (qx.astype(np.float64) * sx[:, None].astype(np.float64)) @ \
        (qw.astype(np.float64) * sw[:, None].astype(np.float64)).T, (qx, sx, qw, sw)


def test_smoothed_product_is_the_same_product():
    """The dequantized smoothed operands reproduce X W^T within the bound their
    quantization steps fix: |sum_k x'w' - x'^q w'^q| <= sum_k |x'| dw + |w'| dx
    + dx dw, with dx = sx/2, dw = sw/2.  A mismatched s (X divided on one
    channel, W multiplied on another) breaks it for most outputs."""
    X = make_activation(16, 512, seed=9, outlier_dims=6).float().numpy()
    W = make_weight(24, 512, 0.02, seed=9).float().numpy()
    a, _ = oracle.channel_absmax(X)
    w, _ = oracle.channel_absmax(W)
    s, _ = oracle.smooth_scales(a, w, 0.5)
    Yq, (qx, sx, qw, sw) = _w8a8(X, W, s)
    Y = X.astype(np.float64) @ W.astype(np.float64).T
    Xs = X.astype(np.float64) / s.astype(np.float64)
    Ws = W.astype(np.float64) * s.astype(np.float64)
    dx, dw = sx.astype(np.float64)[:, None] / 2, sw.astype(np.float64)[None, :] / 2
    bound = (np.abs(Xs).sum(1, keepdims=True) * dw + dx * np.abs(Ws).sum(1)[None, :]
             + X.shape[1] * dx * dw
             + 2.0 ** -22 * (np.abs(Xs) @ np.abs(Ws).T))  # fp32 rounding of X/s and W s
    assert np.all(np.abs(Yq - Y) <= bound)
    # W multiplied on other channels than X is divided on: far outside it
    qw_b, sw_b, _ = oracle.quantize_int8_rows_smoothed(W, np.roll(s, 1))
    Yb = (qx.astype(np.float64) * sx[:, None]) @ (qw_b.astype(np.float64) * sw_b[:, None]).T
    assert np.mean(np.abs(Yb - Y) > bound) > 0.5


def test_smoothing_helps_outlier_activations():
    """Sec. 4.2's point: with a few outlier hidden dims (magnitude 50-100) in X,
    alpha = 0.5 smoothing makes the W8A8 product markedly more accurate than
    plain per-token x per-channel INT8."""
    X = make_activation(64, 1024, seed=11, outlier_dims=6).float().numpy()
    W = make_weight(128, 1024, 0.02, seed=11).float().numpy()
    Y = X.astype(np.float64) @ W.astype(np.float64).T
    a, _ = oracle.channel_absmax(X)
    w, _ = oracle.channel_absmax(W)
    s, _ = oracle.smooth_scales(a, w, 0.5)
    e_plain = np.linalg.norm(_w8a8(X, W)[0] - Y) / np.linalg.norm(Y)
    e_smooth = np.linalg.norm(_w8a8(X, W, s)[0] - Y) / np.linalg.norm(Y)
    assert e_smooth < 0.5 * e_plain, (e_plain, e_smooth)
