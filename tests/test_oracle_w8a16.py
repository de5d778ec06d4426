"""Pins of the W8A16 oracle (8-bit per-channel weights, bf16 activations;
"27届大模型面试准备（十九）…" sec. 2.3 naming table) against other oracle
routines with their own loops and against closed forms."""
import numpy as np
import pytest

import oracle


def bf16_bits_exact(x):
    """bf16 bits of float32 values that bf16 represents exactly."""
    b = oracle.f32_to_bf16(np.asarray(x, np.float32))
    assert np.array_equal(oracle.bf16_to_f32(b), np.asarray(x, np.float32))
    return b


def test_equals_w8a8_when_x_is_scaled_int8():
    """X = 2^-4 qx with int8 qx is exact in bf16; then the W8A16 product is
    the W8A8 product with s_x = 2^-4, bit for bit (every term and the sum
    are exact in binary64)."""
    rng = np.random.default_rng(0)
    M, N, K = 5, 7, 96
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sw = (rng.random(N) * 0.01 + 1e-3).astype(np.float32)
    X = bf16_bits_exact(qx.astype(np.float32) * np.float32(2.0 ** -4))
    Y, st = oracle.gemm_w8a16(X, qw, oracle.W_I8, sw)
    assert st == oracle.OK
    acc, st = oracle.gemm_w8a8_acc(qx, qw)
    ref, _ = oracle.w8a8_rescale(acc, np.full(M, 2.0 ** -4, np.float32), sw)
    np.testing.assert_array_equal(Y, ref)


def test_equals_fp8_product_when_x_is_scaled_e4m3():
    rng = np.random.default_rng(1)
    M, N, K = 4, 6, 64
    qx = rng.integers(0, 256, size=(M, K)).astype(np.uint8)
    qx[(qx & 0x7F) == 0x7F] = 0x38      # no NaN codes
    qw = rng.integers(0, 256, size=(N, K)).astype(np.uint8)
    qw[(qw & 0x7F) == 0x7F] = 0xB8
    sw = (rng.random(N) + 0.5).astype(np.float32)
    X = bf16_bits_exact(oracle.e4m3_to_f32(qx).reshape(M, K) * np.float32(0.125))
    Y, st = oracle.gemm_w8a16(X, qw, oracle.W_E4M3, sw)
    assert st == oracle.OK
    ref, _, st = oracle.gemm_fp8(qx, np.full(M, 0.125, np.float32), qw, sw, 0, M, 0, N)
    assert st == oracle.OK
    np.testing.assert_allclose(Y, ref, rtol=1e-13, atol=1e-300)


def test_equals_w4a16_when_codes_fit_four_bits():
    """int8 codes in [-8, 7] with an fp16-exact row scale are the symmetric
    INT4 codes u = q + 8 with that scale in every group."""
    rng = np.random.default_rng(2)
    M, N, K = 3, 8, 256
    q = rng.integers(-8, 8, size=(N, K)).astype(np.int8)
    s16 = oracle.f32_to_f16((rng.random(N) * 0.05 + 0.01).astype(np.float32))
    sw = oracle.f16_to_f32(s16).astype(np.float32)
    u = (q.astype(np.int16) + 8).astype(np.uint8)
    codes = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    scales = np.repeat(s16.reshape(N, 1), K // 128, axis=1)
    X = oracle.f32_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    Y, st = oracle.gemm_w8a16(X, q, oracle.W_I8, sw)
    ref, st2 = oracle.gemm_w4a16(X, codes, scales, None, 128, True)
    assert st == oracle.OK and st2 == oracle.OK
    np.testing.assert_allclose(Y, ref, rtol=1e-14, atol=1e-14)


def test_unit_codes_give_row_sums():
    rng = np.random.default_rng(3)
    M, K = 4, 40
    x = rng.integers(-50, 50, size=(M, K)).astype(np.float32)
    X = bf16_bits_exact(x)
    for fmt, one in ((oracle.W_I8, 1), (oracle.W_E4M3, 0x38)):   # E4M3 0x38 = 1.0
        qw = np.full((2, K), one, np.uint8)
        Y, st = oracle.gemm_w8a16(X, qw, fmt, np.array([1.0, 2.0], np.float32))
        assert st == oracle.OK
        np.testing.assert_array_equal(Y[:, 0], x.sum(axis=1).astype(np.float64))
        np.testing.assert_array_equal(Y[:, 1], 2.0 * x.sum(axis=1).astype(np.float64))


def test_window_and_arguments():
    rng = np.random.default_rng(4)
    X = oracle.f32_to_bf16(rng.standard_normal((2, 32)).astype(np.float32))
    qw = rng.integers(-127, 128, size=(9, 32)).astype(np.int8)
    sw = np.ones(9, np.float32)
    full, _ = oracle.gemm_w8a16(X, qw, oracle.W_I8, sw)
    part, st = oracle.gemm_w8a16(X, qw, oracle.W_I8, sw, 3, 7)
    assert st == oracle.OK
    np.testing.assert_array_equal(part, full[:, 3:7])
    _, st = oracle.gemm_w8a16(X, qw, 5, sw)
    assert st == oracle.ERR_ARG
    _, st = oracle.gemm_w8a16(X, qw, oracle.W_I8, sw, 4, 10)
    assert st == oracle.ERR_ARG
