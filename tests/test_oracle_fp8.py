"""Pins of the oracle's FP8 E4M3 ("27届大模型面试准备（十九）…" sec. 2.3 names FP8
E4M3 as the 8-bit float format of the newest tensor cores): the code table
against torch's float8_e4m3fn, round-to-nearest-even at every tie, saturation
at 448, subnormals, the per-row quantizer and the exact product."""
import numpy as np
import pytest
import torch

import oracle


def torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def test_decode_table_matches_torch():
    c = np.arange(256, dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_to_f32(c), torch_decode(c), equal_nan=True)


def test_every_finite_value_round_trips():
    c = np.array([i for i in range(256) if (i & 0x7F) != 0x7F], np.uint8)
    v = oracle.e4m3_to_f32(c)
    got = oracle.f32_to_e4m3(v)
    # +0 and -0 keep their sign bits
    assert np.array_equal(got, c)


def test_ties_go_to_the_even_code():
    pos = np.arange(0, 0x7E, dtype=np.uint8)          # 0 .. 446, consecutive codes
    lo, hi = oracle.e4m3_to_f32(pos), oracle.e4m3_to_f32(pos + 1)
    mid = ((lo.astype(np.float64) + hi) / 2).astype(np.float32)   # exact: <= 5 significant bits
    got = oracle.f32_to_e4m3(mid)
    even = np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint8)
    assert np.array_equal(got, even)
    above = np.nextafter(mid, np.float32(np.inf))
    below = np.nextafter(mid, np.float32(0))
    assert np.array_equal(oracle.f32_to_e4m3(above), (pos + 1).astype(np.uint8))
    assert np.array_equal(oracle.f32_to_e4m3(below), pos)


def test_matches_torch_rounding_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 20000),
                        rng.standard_normal(20000) * 0.05,
                        rng.standard_normal(5000) * 1e-3]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f32_to_e4m3(x), ref)


@pytest.mark.parametrize("x,code", [(448.0, 0x7E), (449.0, 0x7E), (463.9, 0x7E), (1e6, 0x7E),
                                    (-500.0, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -10, 0x00),
                                    (3 * 2.0 ** -10, 0x02), (2.0 ** -6, 0x08), (1.0, 0x38),
                                    (1.0625, 0x38), (1.1875, 0x3A)])
def test_hand_codes(x, code):
    assert int(oracle.f32_to_e4m3([x])[0]) == code


def test_row_quantizer():
    W = np.array([[448.0, -224.0, 1.0, 0.0], [0.0, 0.0, 0.0, 0.0], [-0.5, 0.25, 0.125, 0.0625]],
                 np.float32)
    q, s, st = oracle.quantize_fp8_rows(W)
    assert st == oracle.OK
    assert s.tolist() == [1.0, np.float32(1e-8), np.float32(np.float32(0.5) / np.float32(448.0))]
    assert q[0].tolist() == [0x7E, 0xF6, 0x38, 0x00]     # 448, -224, 1, 0
    assert q[1].tolist() == [0, 0, 0, 0]
    assert int(q[2, 0]) == 0xFE                          # the row maximum maps to -448


def test_product_is_exact_against_torch_fp8_values():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((5, 96)).astype(np.float32)
    W = (rng.standard_normal((7, 96)) * 0.02).astype(np.float32)
    qx, sx, _ = oracle.quantize_fp8_rows(X)
    qw, sw, _ = oracle.quantize_fp8_rows(W)
    Y, acc, st = oracle.gemm_fp8(qx, sx, qw, sw, 0, 5, 0, 7)
    assert st == oracle.OK
    ref_acc = torch_decode(qx).astype(np.float64) @ torch_decode(qw).astype(np.float64).T
    assert np.array_equal(acc, ref_acc)
    np.testing.assert_allclose(Y, ref_acc * sx[:, None] * sw[None, :], rtol=1e-15)


def test_fp8_more_accurate_than_int8_on_outlier_activations():
    """Sec. 2.3 calls FP8 the most accurate 8-bit scheme: with per-token x
    per-channel scales on activations with outlier dims, the E4M3 product is
    closer to the fp64 product than the INT8 one."""
    from workloads import make_activation, make_weight
    X = make_activation(128, 1024, seed=11, outlier_dims=6).float().numpy()
    W = make_weight(256, 1024, 0.02, seed=11, outlier_frac=0.001, outlier_scale=30.0).float().numpy()
    Y = X.astype(np.float64) @ W.astype(np.float64).T
    qx, sx, _ = oracle.quant_act_i8(X)
    qw, sw, _ = oracle.quantize_int8_rows(W)
    Yi = (qx * sx[:, None].astype(np.float64)) @ (qw * sw[:, None].astype(np.float64)).T
    fx, fsx, _ = oracle.quantize_fp8_rows(X)
    fw, fsw, _ = oracle.quantize_fp8_rows(W)
    Yf, _, _ = oracle.gemm_fp8(fx, fsx, fw, fsw, 0, 128, 0, 256)
    e_int8 = np.linalg.norm(Yi - Y) / np.linalg.norm(Y)
    e_fp8 = np.linalg.norm(Yf - Y) / np.linalg.norm(Y)
    assert e_fp8 < 0.75 * e_int8, (e_int8, e_fp8)
