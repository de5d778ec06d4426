"""Pins of the oracle's GPTQ ("27届大模型面试准备（十九）…" sec. 4.3): the damped
inverse-Hessian factor on a hand case and as an identity, GPTQ with an
identity factor equal to plain round-to-nearest, errors pushed only forward,
and the page's claim that GPTQ lowers the layer's reconstruction error."""
import numpy as np
import pytest

import oracle


def test_factor_hand_case():
    X = np.array([[1.0, 0.0], [0.0, 2.0]], np.float32)       # H = diag(2, 8), mean 5
    U, st = oracle.gptq_hinv_chol(X, 0.01)
    assert st == oracle.OK
    np.testing.assert_allclose(U, np.diag([1 / np.sqrt(2.05), 1 / np.sqrt(8.05)]), rtol=1e-14)


def test_factor_inverts_the_damped_hessian():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((64, 24)).astype(np.float32)
    X[:, 5] = X[:, 3] * 0.9 + 0.1 * X[:, 5]                  # correlated inputs
    U, st = oracle.gptq_hinv_chol(X, 0.01)
    assert st == oracle.OK
    assert np.allclose(np.tril(U, -1), 0.0)
    H = 2.0 * X.astype(np.float64).T @ X.astype(np.float64)
    H += 0.01 * np.mean(np.diag(H)) * np.eye(24)
    np.testing.assert_allclose(U.T @ U @ H, np.eye(24), atol=1e-9)


def _rtn(W, sym):
    return oracle.quantize_int4(W, 128, sym)


@pytest.mark.parametrize("sym", [True, False])
def test_identity_factor_is_round_to_nearest(sym):
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((16, 384)) * 0.02).astype(np.float32)
    c, s, z, st = oracle.gptq_quantize(W, np.eye(384), 128, sym)
    assert st == oracle.OK
    rc, rs, rz, _ = _rtn(W, sym)
    assert np.array_equal(c, rc) and np.array_equal(s, rs)
    if not sym:
        assert np.array_equal(z, rz)


def test_errors_move_only_forward():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((256, 256)).astype(np.float32)
    U, _ = oracle.gptq_hinv_chol(X, 0.01)
    W = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
    c0, s0, _, _ = oracle.gptq_quantize(W, U, 128, True)
    W2 = W.copy()
    W2[:, 200:] += 0.05                                       # columns of the second group
    c1, s1, _, _ = oracle.gptq_quantize(W2, U, 128, True)
    # the first group (columns 0..127, bytes 0..63) cannot see them
    assert np.array_equal(c0[:, :64], c1[:, :64]) and np.array_equal(s0[:, 0], s1[:, 0])
    assert not np.array_equal(c0[:, 64:], c1[:, 64:])


def _recon_err(X, W, codes, scales, zeros, sym):
    What, _ = oracle.dequant_int4(codes, scales, zeros, W.shape[1], 128, sym)
    d = X.astype(np.float64) @ (W.astype(np.float64) - What.astype(np.float64)).T
    return np.linalg.norm(d)


@pytest.mark.parametrize("sym", [True, False])
def test_gptq_lowers_reconstruction_error(sym):
    """Sec. 4.3's objective ||X W^T - X W_hat^T||: with correlated calibration
    activations GPTQ beats round-to-nearest with the same format."""
    rng = np.random.default_rng(3)
    base = rng.standard_normal((512, 32))
    X = (base @ rng.standard_normal((32, 256)) + 0.1 * rng.standard_normal((512, 256))).astype(np.float32)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    U, st = oracle.gptq_hinv_chol(X, 0.01)
    assert st == oracle.OK
    g = oracle.gptq_quantize(W, U, 128, sym)
    r = _rtn(W, sym)
    e_gptq = _recon_err(X, W, g[0], g[1], g[2], sym)
    e_rtn = _recon_err(X, W, r[0], r[1], r[2], sym)
    assert e_gptq < 0.8 * e_rtn, (e_gptq, e_rtn)
