"""Host restatement of the CUDA-core decode kernel's arithmetic (W4A16,
M <= 4): each (activation row, 128-group) of X becomes integers
x' = rint(x 2^e) with the group's max |x'| in [2^12, 2^13), which fit the
signed 16-bit halves of DP2A.  A code word's even nibbles (w & 0x0F0F0F0F)
and sixteen times its odd ones (w & 0xF0F0F0F0) are taken against them in two
integer sums per row and lane; the group's dot product is an exact integer,
scaled once by s 2^-e.  These tests pin the operand ranges DP2A needs, the
exactness and size of the integer sums and the error bound against the fp64
product."""
import numpy as np
import pytest
import torch

import oracle
from workloads import bf16_bits, make_activation, make_weight


def prepare(x):
    """x: float32 [G, 128] (bf16 values) -> (x' int64, e int)."""
    amax = np.abs(x).max(axis=1).astype(np.float32)
    E = (amax.view(np.uint32) >> 23).astype(np.int64)
    e = np.clip(139 - E, -126, 126)
    xi = np.rint(x.astype(np.float64) * np.exp2(e)[:, None]).astype(np.int64)
    return xi, e


def magic_round(x, e):
    """fma(x, 2^e, 1.5 2^23) in binary32, as the kernel computes x': the bit
    pattern minus that of 1.5 2^23."""
    prod = (x.astype(np.float64) * np.exp2(e)[:, None]).astype(np.float32)   # exact (power of 2)
    r = (prod + np.float32(12582912.0)).astype(np.float32)                    # one rounding, RNE
    return r.view(np.uint32).astype(np.int64) - 0x4B400000


def test_operands_fit_dp2a():
    rng = np.random.default_rng(0)
    for scale in (1e-6, 1e-2, 1.0, 50.0, 3e4):
        x = oracle.bf16_to_f32(oracle.f32_to_bf16(
            (rng.standard_normal((400, 128)) * scale).astype(np.float32))).reshape(400, 128)
        xi, e = prepare(x)
        m = np.abs(xi).max(axis=1)
        assert ((m >= 2 ** 12) & (m <= 2 ** 13)).all()   # the rounded max may reach 2^13
        assert xi.min() >= -2 ** 15 and xi.max() < 2 ** 15   # signed 16-bit halves
        # the fma with 1.5 2^23 rounds to the same integers (ties to even)
        assert np.array_equal(magic_round(x, e), xi)
        # its low 16 bits are x' as a two's-complement 16-bit value
        lo = (magic_round(x, e) + 0x4B400000) & 0xFFFF
        assert np.array_equal(np.where(lo >= 2 ** 15, lo - 2 ** 16, lo), xi)


def test_integer_sums_are_exact_and_small():
    rng = np.random.default_rng(1)
    x = oracle.bf16_to_f32(oracle.f32_to_bf16(rng.standard_normal((200, 128)).astype(np.float32))).reshape(200, 128)
    xi, _ = prepare(x)
    # extreme operands: every code 15 against the largest |x'| everywhere
    u = rng.integers(0, 16, (200, 128))
    z = rng.integers(0, 16, (200, 1))
    worst_even = 16 * 15 * 2 ** 13          # one lane: 16 even elements
    worst_odd = 16 * (16 * 15) * 2 ** 13    # 16 odd elements, codes x 16
    assert worst_even < 2 ** 31 and worst_odd < 2 ** 31
    ev = (u[:, 0:32:2] * xi[:, 0:32:2]).sum(1)
    od16 = ((16 * u[:, 1:32:2]) * xi[:, 1:32:2]).sum(1)
    assert (od16 % 16 == 0).all()            # the odd sum divides exactly by 16
    lane = ev + od16 // 16
    assert np.array_equal(lane, (u[:, :32] * xi[:, :32]).sum(1))
    # the group's sum minus the zero point's share is exact below 2^24, so
    # its conversion to binary32 is exact too
    t = (u * xi).sum(1) - z[:, 0] * xi.sum(1)
    assert np.array_equal(t, ((u - z) * xi).sum(1))
    assert 15 * 128 * 2 ** 13 < 2 ** 24


@pytest.mark.parametrize("sym", [True, False])
def test_product_error_within_the_stated_bound(sym):
    """Only elements below 2^-5 of their group maximum lose bits, each by at
    most 2^-13 of the maximum (a group holding an outlier dimension rounds
    nearly all its other elements); the product stays inside the 2e-3
    row-normalised tolerance against the fp64 oracle with a wide margin."""
    N, K, M = 64, 1024, 2
    W = make_weight(N, K, 0.02, seed=4, outlier_frac=0.01, outlier_scale=30.0, dtype=torch.float32)
    codes, scales, zeros, st = oracle.quantize_int4(W.numpy(), 128, sym)
    assert st == oracle.OK
    X = make_activation(M, K, seed=5, outlier_dims=6)
    Xb = bf16_bits(X)
    ref, _ = oracle.gemm_w4a16(Xb, codes, scales, zeros, 128, sym)
    x = oracle.bf16_to_f32(Xb).reshape(M, K)
    u = np.zeros((N, K), np.int64)
    u[:, 0::2] = codes & 15
    u[:, 1::2] = codes >> 4
    s = oracle.f16_to_f32(scales).reshape(N, K // 128).astype(np.float32)
    zf = np.full((N, K // 128), 8) if sym else oracle.f16_to_f32(zeros).reshape(N, K // 128)
    Y = np.zeros((M, N))
    for m in range(M):
        xi, e = prepare(x[m].reshape(K // 128, 128))
        for g in range(K // 128):
            ug = u[:, g * 128:(g + 1) * 128] - zf[:, g:g + 1].astype(np.int64)
            t = (ug * xi[g]).sum(1)                       # exact integers
            Y[m] += (t.astype(np.float32) * (s[:, g] * np.float32(2.0 ** -e[g]))).astype(np.float64)
    err = np.abs(Y - ref).max(axis=1) / np.linalg.norm(ref, axis=1)
    assert err.max() < 1e-3


def test_exact_down_to_two_to_the_minus_five_of_the_maximum():
    rng = np.random.default_rng(2)
    x = oracle.bf16_to_f32(oracle.f32_to_bf16(rng.standard_normal((2000, 128)).astype(np.float32))).reshape(2000, 128)
    xi, e = prepare(x)
    amax = np.abs(x).max(axis=1, keepdims=True)
    err = np.abs(x - xi * np.exp2(-e)[:, None])
    assert (err[np.abs(x) >= amax * 2.0 ** -5] == 0).all()
    assert (err <= amax * 2.0 ** -13).all()
    assert (err > 0).any()


@pytest.mark.parametrize("N,K,M", [(136, 192, 1), (264, 4160, 4), (512, 4096, 2)])
def test_w8a16_int8_fixed_point_x(N, K, M):
    """The W8A16 decode with int8 codes reads X the same way: per activation
    row and 128-element group, x' = rint(x 2^e) (the magic-constant rounding);
    a lane's 16 codes times x' (two signed DP2A per code word) is an exact
    integer below 2^24, scaled by 2^-e.  On weights with outlier rows and
    activations with six outlier dims the product stays well inside the
    2e-3 row bound against the fp64 oracle."""
    W = make_weight(N, K, 0.02, seed=N + K, outlier_frac=0.02, outlier_scale=20.0).float().numpy()
    s = np.maximum(np.abs(W).max(axis=1) / np.float32(127), np.float32(1e-8)).astype(np.float32)
    q = np.clip(np.rint(W / s[:, None]), -127, 127).astype(np.int64)
    X = make_activation(M, K, seed=M + K, outlier_dims=6)
    x = X.float().numpy()
    Y = np.zeros((M, N))
    for g0 in range(0, K, 128):
        xg = x[:, g0:g0 + 128]
        xi, e = prepare(xg)
        assert np.abs(xi).max() <= 2 ** 13                      # signed 16-bit DP2A operand
        np.testing.assert_array_equal(magic_round(xg, e), xi)   # the kernel's rounding
        for l0 in range(0, xg.shape[1], 16):                    # one lane's 16 codes
            isum = xi[:, l0:l0 + 16] @ q[:, g0 + l0:g0 + l0 + 16].T
            assert np.abs(isum).max() < 2 ** 24                 # exact in binary32
            Y += isum * np.exp2(-e)[:, None]
    Y *= s[None, :]
    Yref, st = oracle.gemm_w8a16(bf16_bits(X), q.astype(np.int8), oracle.W_I8, s)
    assert st == oracle.OK
    err = np.abs(Y - Yref).max(axis=1) / np.linalg.norm(Yref, axis=1)
    assert err.max() <= 5e-4, err.max()
