"""Pins for the oracle's IEEE-754 conversions and rounding.

The oracle writes fp16 / bf16 rounding from the format definitions; here it is
checked against two independent implementations of the same standard: numpy's
float16 cast and torch's bfloat16 cast (both round to nearest even), over every
16-bit pattern and over edge and random binary32 inputs.
"""
import numpy as np
import pytest
import torch

import oracle


def _edge_f32():
    vals = [0.0, -0.0, 1.0, -1.0, 0.5, 65504.0, 65519.99, 65520.0, 65536.0, 1e6,
            6.1035156e-05, 6.0975552e-05, 5.9604645e-08, 2.9802322e-08,
            2.9802326e-08, 1e-8, 1e-30, 3.4e38, -3.4e38, np.inf, -np.inf,
            1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2048.0 + 1.0, 2048.0 + 3.0,
            1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.1754944e-38, 1e-40, 1e-45]
    return np.array(vals, dtype=np.float32)


def _random_f32(n=200_000, seed=0):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    y = (rng.standard_normal(n) * 10.0 ** rng.uniform(-9, 6, n)).astype(np.float32)
    return np.concatenate([x, y, _edge_f32()])


def _bits_equal_with_nan(a_bits, b_bits, a_f, b_f):
    both_nan = np.isnan(a_f) & np.isnan(b_f)
    return np.all((a_bits == b_bits) | both_nan)


def test_f32_to_f16_matches_numpy():
    x = _random_f32()
    ours = oracle.f32_to_f16(x)
    ref = x.astype(np.float16).view(np.uint16)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"first mismatch x={x[bad[0]]!r} ours={ours[bad[0]]:#06x} ref={ref[bad[0]]:#06x}"


def test_f32_to_f16_nan():
    ours = oracle.f32_to_f16(np.array([np.nan], np.float32))
    assert (ours[0] & 0x7C00) == 0x7C00 and (ours[0] & 0x3FF) != 0


def test_f16_to_f32_all_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    assert _bits_equal_with_nan(ours.view(np.uint32), ref.view(np.uint32), ours, ref)


def test_f32_to_bf16_matches_torch():
    x = _random_f32(seed=1)
    ours = oracle.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"first mismatch x={x[bad[0]]!r} ours={ours[bad[0]]:#06x} ref={ref[bad[0]]:#06x}"


def test_bf16_to_f32_all_patterns():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f32(b)
    ref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert _bits_equal_with_nan(ours.view(np.uint32), ref.view(np.uint32), ours, ref)


@pytest.mark.parametrize("v,expect", [(0.5, 0.0), (1.5, 2.0), (2.5, 2.0), (-0.5, -0.0),
                                      (-1.5, -2.0), (-2.5, -2.0), (3.5, 4.0),
                                      (2.4999998, 2.0), (7.5, 8.0), (-7.5, -8.0)])
def test_round_half_even_ties(v, expect):
    assert oracle.round_half_even(v) == expect


def test_round_half_even_matches_numpy_round():
    # numpy.round / numpy.rint round half to even, as the pages' numpy code does
    rng = np.random.default_rng(3)
    v = (rng.integers(-40, 40, 5000) / 2.0).astype(np.float32)
    v = np.concatenate([v, rng.standard_normal(5000).astype(np.float32) * 20])
    ours = np.array([oracle.round_half_even(float(a)) for a in v], np.float32)
    assert np.array_equal(ours, np.round(v))
