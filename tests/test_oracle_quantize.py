"""Pins for the oracle's quantizers, dequantizer and products.

Each check rests on something other than the oracle's own formulas: values the
pages print (tests/golden/worked_examples.json, with citations), hand-worked
groups whose scales are exact binary fractions, closed forms for the metadata
size, the nearest-grid-point property checked by brute force over all 16
codes, numpy matrix products and exact Python/numpy integer sums.
"""
import json
import os

import numpy as np
import pytest

import oracle
from workloads import make_weight, make_activation, bf16_bits

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "worked_examples.json")))


def _group(values, g=128, fill=0.0):
    row = np.full((1, g), fill, np.float32)
    row[0, :len(values)] = values
    return row


def _unpack(codes, K):
    lo = codes & 0x0F
    hi = codes >> 4
    out = np.empty((codes.shape[0], K), np.int32)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


# ---------------------------------------------------------------- hand-worked

def test_symmetric_hand_worked_group():
    # amax = 1.75 -> s = 1.75 / 7 = 0.25 exactly (also exact in fp16)
    vals = [-1.75, 0.5, 1.75, 0.125, 0.375, 0.625, -0.375, 0.0, -0.25]
    codes, scales, zeros, st = oracle.quantize_int4(_group(vals), 128, sym=True)
    assert st == oracle.OK and zeros is None
    assert oracle.f16_to_f32(scales)[0, 0] == 0.25
    q = _unpack(codes, 128)[0, :len(vals)] - 8
    # 0.125/0.25 = 0.5 -> 0, 0.375/0.25 = 1.5 -> 2, 0.625/0.25 = 2.5 -> 2 (half to even)
    assert list(q) == [-7, 2, 7, 0, 2, 2, -2, 0, -1]
    xh, _ = oracle.dequant_int4(codes, scales, zeros, 128, 128, sym=True)
    assert list(xh[0, :len(vals)]) == [-1.75, 0.5, 1.75, 0.0, 0.5, 0.5, -0.5, 0.0, -0.25]


def test_asymmetric_hand_worked_group():
    # range [-0.5, 1.0]: s32 = 1.5/15 = 0.1 (fp32), stored fp16 0.0999755859375,
    # z = round(0.5 / 0.0999755859375) = round(5.0012...) = 5
    vals = [-0.5, 1.0, 0.3, 0.0, -0.2]
    codes, scales, zeros, st = oracle.quantize_int4(_group(vals, fill=0.0), 128, sym=False)
    assert st == oracle.OK
    s = oracle.f16_to_f32(scales)[0, 0]
    assert s == np.float32(0.0999755859375)
    assert oracle.f16_to_f32(zeros)[0, 0] == 5.0
    q = _unpack(codes, 128)[0, :len(vals)]
    # round(x/s) + z: -0.5 -> -5+5=0, 1.0 -> 10+5=15, 0.3 -> 3+5=8, 0 -> 5, -0.2 -> -2+5=3
    assert list(q) == [0, 15, 8, 5, 3]


def test_round_then_add_reading_on_odd_zero_point():
    # A tie x/s = 2.5 with odd z = 3: round(x/s) + z = 2 + 3 = 5, whereas
    # round(x/s + z) = round(5.5) = 6.  The oracle follows round-then-add.
    # min = -0.75, max = 3.0 -> s = 3.75/15 = 0.25, z = round(0.75/0.25) = 3.
    vals = [-0.75, 3.0, 0.625]
    codes, scales, zeros, st = oracle.quantize_int4(_group(vals), 128, sym=False)
    assert oracle.f16_to_f32(scales)[0, 0] == 0.25
    assert oracle.f16_to_f32(zeros)[0, 0] == 3.0
    q = _unpack(codes, 128)[0, :3]
    assert list(q) == [0, 15, 5]


def test_per_tensor_outlier_worked_example():
    ex = GOLDEN["per_tensor_int8_outlier"]
    row = np.zeros((1, 64), np.float32)
    row[0, 0] = ex["amax"]
    row[0, 1] = ex["x"]
    q, s, st = oracle.quantize_int8_rows(row)
    assert st == oracle.OK
    assert abs(s[0] - ex["scale_printed"]) < 5e-4
    assert q[0, 1] == ex["q_printed"] and q[0, 0] == ex["qmax"]
    xh, _ = oracle.dequant_int8_rows(q, s)
    assert abs(xh[0, 1] - ex["x_hat_printed"]) < 5e-4
    rel = abs(xh[0, 1] - ex["x"]) / ex["x"]
    assert abs(rel - ex["relative_error_printed"]) < 0.01


def test_per_token_act_quant_hand_worked():
    # amax = 31.75 -> s = 31.75/127 = 0.25 exactly
    x = np.array([[-31.75, 0.375, 0.625, 0.125, 31.75, -0.125]], np.float32)
    q, s, st = oracle.quant_act_i8(x)
    assert st == oracle.OK and s[0] == 0.25
    assert list(q[0]) == [-127, 2, 2, 0, 127, 0]
    zero = np.zeros((1, 16), np.float32)
    q0, s0, _ = oracle.quant_act_i8(zero)
    assert s0[0] == np.float32(1e-8) and not q0.any()


# ----------------------------------------------------------- degenerate groups

def test_degenerate_symmetric_group_is_zero():
    codes, scales, zeros, st = oracle.quantize_int4(np.zeros((1, 128), np.float32), 128, True)
    assert st == oracle.OK
    assert (_unpack(codes, 128) == 8).all()          # q = 0 stored as u = 8
    assert oracle.f16_to_f32(scales)[0, 0] == 0.0    # scale = amax = 0
    xh, _ = oracle.dequant_int4(codes, scales, zeros, 128, 128, True)
    assert not xh.any()


def test_degenerate_asymmetric_group_follows_page_rule():
    # constant group: max - min < 1e-8 -> q = 0, s = 1.0, z = 0
    codes, scales, zeros, st = oracle.quantize_int4(np.full((1, 128), 0.3, np.float32), 128, False)
    assert (_unpack(codes, 128) == 0).all()
    assert oracle.f16_to_f32(scales)[0, 0] == 1.0 and oracle.f16_to_f32(zeros)[0, 0] == 0.0


def test_scale_underflowing_fp16_is_degenerate():
    # amax = 1e-7: amax/7 rounds to fp16 zero -> treated as a degenerate range
    g = np.zeros((1, 128), np.float32)
    g[0, 3] = 1e-7
    codes, scales, _, _ = oracle.quantize_int4(g, 128, True)
    assert (_unpack(codes, 128) == 8).all()


def test_nonfinite_input_reports_status():
    g = np.zeros((1, 128), np.float32)
    g[0, 5] = np.inf
    assert oracle.quantize_int4(g, 128, True)[3] == oracle.ERR_NONFINITE
    assert oracle.quant_act_i8(g)[2] == oracle.ERR_NONFINITE


# --------------------------------------------------------------- invariants

@pytest.fixture(scope="module")
def random_weight():
    W = make_weight(48, 1024, 0.02, seed=5, outlier_frac=0.004, outlier_scale=30.0)
    return W, bf16_bits(W), W.float().numpy()


@pytest.mark.parametrize("sym", [True, False])
def test_codes_are_nearest_grid_points(random_weight, sym):
    """Brute force over all 16 codes: the chosen code's grid point is the
    nearest to x (up to the fp32 rounding of x/s), and the range holds."""
    _, bits, Wf = random_weight
    N, K = Wf.shape
    codes, scales, zeros, st = oracle.quantize_int4(bits, 128, sym, dtype_tag=oracle.BF16)
    assert st == oracle.OK
    u = _unpack(codes, K)
    s = np.repeat(oracle.f16_to_f32(scales).astype(np.float64), 128, axis=1)
    if sym:
        zeff = np.full_like(s, 8.0)
    else:
        z = oracle.f16_to_f32(zeros)
        assert ((z >= 0) & (z <= 15) & (z == np.round(z))).all()
        zeff = np.repeat(z.astype(np.float64), 128, axis=1)
    grid = s[..., None] * (np.arange(16)[None, None, :] - zeff[..., None])
    err_all = np.abs(Wf.astype(np.float64)[..., None] - grid)
    chosen = np.take_along_axis(err_all, u[..., None], axis=2)[..., 0]
    best = err_all.min(axis=2)
    assert (chosen <= best + 1e-6 * s).all()


def test_half_step_bound_in_straddling_groups(random_weight):
    _, bits, Wf = random_weight
    N, K = Wf.shape
    for sym in (True, False):
        codes, scales, zeros, _ = oracle.quantize_int4(bits, 128, sym, dtype_tag=oracle.BF16)
        xh, _ = oracle.dequant_int4(codes, scales, zeros, K, 128, sym)
        s = oracle.f16_to_f32(scales)
        G = K // 128
        for n in range(N):
            for g in range(G):
                x = Wf[n, g * 128:(g + 1) * 128].astype(np.float64)
                if not (x.min() <= 0.0 <= x.max()):
                    continue
                err = np.abs(x - xh[n, g * 128:(g + 1) * 128])
                # half a step, plus the fp16 rounding of s (half an fp16 ulp per code step)
                slack = 8 * s[n, g] * 2.0 ** -11
                assert err.max() <= s[n, g] / 2 + slack, (n, g, err.max(), s[n, g])


def test_symmetric_zero_point_is_absent_and_codes_in_range(random_weight):
    _, bits, _ = random_weight
    codes, scales, zeros, _ = oracle.quantize_int4(bits, 128, True, dtype_tag=oracle.BF16)
    q = _unpack(codes, 1024) - 8
    assert zeros is None and q.min() >= -8 and q.max() <= 7


# ------------------------------------------------------------- closed forms

def test_metadata_overhead_closed_forms():
    ex = GOLDEN["group128_effective_bits"]
    K, g = ex["in_features"], ex["group_size"]
    W = np.random.default_rng(0).standard_normal((8, K)).astype(np.float32)
    codes, scales, zeros, _ = oracle.quantize_int4(W, g, sym=False)
    assert scales.shape[1] == ex["groups_per_row_printed"]
    meta_bits = 8 * (scales.nbytes + zeros.nbytes) / W.size
    payload_bits = 8 * codes.nbytes / W.size
    assert payload_bits == 4.0
    assert payload_bits + meta_bits == ex["effective_bits_printed"]
    share = GOLDEN["metadata_share"]
    for gs, printed in ((128, share["share_g128_printed"]), (32, share["share_g32_printed"])):
        c, s, _, _ = oracle.quantize_int4(W, gs, sym=True)
        ratio = s.nbytes / c.nbytes
        assert abs(ratio - printed) < 0.001


# ------------------------------------------------------------------- products

def test_gemm_w4a16_matches_numpy_product():
    W = make_weight(24, 256, 0.02, seed=9, outlier_frac=0.01, outlier_scale=20.0)
    X = make_activation(3, 256, seed=10)
    for sym in (True, False):
        codes, scales, zeros, _ = oracle.quantize_int4(bf16_bits(W), 128, sym, oracle.BF16)
        xh, _ = oracle.dequant_int4(codes, scales, zeros, 256, 128, sym)
        Y, st = oracle.gemm_w4a16(bf16_bits(X), codes, scales, zeros, 128, sym)
        ref = X.double().numpy() @ xh.astype(np.float64).T
        assert st == oracle.OK
        np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12)
        Yw, _ = oracle.gemm_w4a16(bf16_bits(X), codes, scales, zeros, 128, sym, n0=5, n1=11)
        np.testing.assert_array_equal(Yw, Y[:, 5:11])


def test_gemm_w4a16_hand_worked_row():
    # one row: all codes q = 1 with s = 0.25 in group 0, q = -2 with s = 0.5 in
    # group 1; X = all ones -> Y = 128*0.25 + 128*(-1.0) = -96
    row = np.concatenate([np.full(128, 0.25), np.full(128, -1.0)]).astype(np.float32)
    row[0] = 1.75
    row[128] = -3.5
    codes, scales, zeros, _ = oracle.quantize_int4(row[None, :], 128, True)
    ones = np.full((1, 256), 0x3F80, np.uint16)  # bf16 1.0
    Y, _ = oracle.gemm_w4a16(ones, codes, scales, None, 128, True)
    assert Y[0, 0] == 127 * 0.25 + 1.75 + 127 * -1.0 - 3.5


def test_w8a8_accumulator_exact_and_overflow():
    rng = np.random.default_rng(4)
    qx = rng.integers(-128, 128, (5, 300)).astype(np.int8)
    qw = rng.integers(-127, 128, (7, 300)).astype(np.int8)
    acc, st = oracle.gemm_w8a8_acc(qx, qw)
    assert st == oracle.OK
    exact = [[sum(int(a) * int(b) for a, b in zip(qx[m], qw[n])) for n in range(7)]
             for m in range(5)]
    assert acc.tolist() == exact
    sub, _ = oracle.gemm_w8a8_acc(qx, qw, 1, 4, 2, 6)
    assert sub.tolist() == [r[2:6] for r in exact[1:4]]
    big = np.full((1, 140_000), 127, np.int8)
    _, st = oracle.gemm_w8a8_acc(big, big)
    assert st == oracle.ERR_OVERFLOW


def test_w8a8_rescale():
    acc = np.array([[3, -4]], np.int32)
    Y, _ = oracle.w8a8_rescale(acc, np.array([0.5], np.float32), np.array([2.0, 0.25], np.float32))
    assert Y.tolist() == [[3.0, -0.5]]
