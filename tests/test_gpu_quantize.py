"""GPU parity of the quantize / pack / dequantize / per-row INT8 kernels:
bit-exact against the CPU oracle on the same seeded inputs, at the workloads'
full sizes and on small, ragged and degenerate cases."""
import numpy as np
import pytest
import torch

import bit_gemm_group_b200 as wq
import oracle
from parity_util import oracle_input, u16
from workloads import WORKLOADS, bf16_bits, make_weight, make_activation

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    wq.wq_get_device_status(reset=True)
    yield
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK


def check_int4(W: torch.Tensor, g: int, sym: bool):
    codes, scales, zeros = wq.quantize_pack(W.cuda(), g, 4, sym)
    arr, tag = oracle_input(W)
    oc, osc, oz, st = oracle.quantize_int4(arr, g, sym, dtype_tag=tag)
    assert st == oracle.OK
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)
    np.testing.assert_array_equal(u16(scales), osc)
    if not sym:
        np.testing.assert_array_equal(u16(zeros), oz)
    # dequantize both ways: fp32 exact, bf16 = round-to-nearest-even of it
    K = W.shape[1]
    ref, _ = oracle.dequant_int4(oc, osc, oz, K, g, sym)
    d32 = wq.dequant(codes, scales, zeros, K, g, 4, sym, torch.float32)
    np.testing.assert_array_equal(d32.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    d16 = wq.dequant(codes, scales, zeros, K, g, 4, sym, torch.bfloat16)
    np.testing.assert_array_equal(u16(d16), oracle.f32_to_bf16(ref))
    return codes, scales, zeros


def test_tiny_workload():
    wl = WORKLOADS["tiny"]
    check_int4(wl.weight(0), 128, wl.sym)


@pytest.mark.parametrize("i", [0, 1, 2])
def test_7b_shapes_symmetric(i):
    wl = WORKLOADS["7b-decode"]
    check_int4(wl.weight(i), 128, True)


@pytest.mark.parametrize("i", [0, 1])
def test_70b_shapes_asymmetric(i):
    wl = WORKLOADS["70b-decode"]
    check_int4(wl.weight(i), 128, False)


def test_prefill_weight():
    wl = WORKLOADS["prefill"]
    check_int4(wl.weight(0), 128, True)


@pytest.mark.parametrize("N,K", [(1, 128), (8, 128), (24, 256), (136, 384), (3, 1024)])
@pytest.mark.parametrize("sym", [True, False])
def test_small_and_ragged(N, K, sym):
    W = make_weight(N, K, 0.02, seed=N * 7 + K, outlier_frac=0.01, outlier_scale=25.0)
    check_int4(W, 128, sym)


@pytest.mark.parametrize("g", [32, 64, 256, 1024])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_group_sizes_and_dtypes(g, dtype):
    W = make_weight(40, 2048, 0.05, seed=g, outlier_frac=0.002, outlier_scale=10.0, dtype=dtype)
    check_int4(W, g, sym=True)
    check_int4(W, g, sym=False)


def test_ties_and_degenerate_groups():
    K = 512
    W = torch.zeros(6, K)
    # row 0 group 0: s = 0.25 exactly, values on .5 ties of x/s
    W[0, :8] = torch.tensor([-1.75, 1.75, 0.125, 0.375, 0.625, -0.375, -0.125, 0.875])
    # row 0 group 1: asym tie with odd zero point (min -0.75, max 3.0 -> s 0.25, z 3)
    W[0, 128:131] = torch.tensor([-0.75, 3.0, 0.625])
    # row 1: constant groups (asym degenerate) and an all-zero group
    W[1, :128] = 0.3
    W[1, 128:256] = -2.0
    # row 2: scale underflows fp16
    W[2, 5] = 1e-7
    # row 3: group entirely positive / entirely negative (z clipped)
    W[3, :128] = torch.linspace(0.5, 1.5, 128)
    W[3, 128:256] = torch.linspace(-1.5, -0.5, 128)
    # row 4: huge and tiny magnitudes
    W[4, :128] = torch.linspace(-1000.0, 1000.0, 128)
    W[4, 128:256] = torch.linspace(-1e-5, 1e-5, 128)
    W[5] = torch.randn(K, generator=torch.Generator().manual_seed(0))
    for sym in (True, False):
        check_int4(W, 128, sym)
        check_int4(W.to(torch.bfloat16), 128, sym)


def test_nonfinite_input_sets_device_status():
    W = torch.zeros(4, 256)
    W[2, 7] = float("inf")
    W[3, 9] = float("nan")
    wq.quantize_pack(W.cuda(), 128, 4, True)
    assert wq.wq_get_device_status(reset=True) == wq.WQ_ERR_NONFINITE
    q = torch.empty(4, 256, dtype=torch.int8, device="cuda")
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    wq.wq_quant_act_i8(W.to(torch.bfloat16).cuda(), q, s)
    assert wq.wq_get_device_status(reset=True) == wq.WQ_ERR_NONFINITE


def test_deterministic():
    W = WORKLOADS["7b-decode"].weight(0).cuda()
    a = wq.quantize_pack(W, 128, 4, True)
    b = wq.quantize_pack(W, 128, 4, True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ------------------------------------------------------------------ INT8 rows

def check_int8_rows(W):
    q, s, _ = wq.quantize_pack(W.cuda(), W.shape[1], 8, True)
    arr, tag = oracle_input(W)
    oq, os_, st = oracle.quantize_int8_rows(arr, dtype_tag=tag)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    ref, _ = oracle.dequant_int8_rows(oq, os_)
    d = wq.dequant(q, s, None, W.shape[1], W.shape[1], 8, True, torch.float32)
    np.testing.assert_array_equal(d.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_w8a8_weight_per_channel():
    check_int8_rows(WORKLOADS["w8a8"].weight(0))


def test_int8_rows_edge():
    W = make_weight(5, 48, 0.02, seed=3, dtype=torch.float32)
    W[1] = 0.0
    W[2, 0] = 100.0
    W[2, 1] = 0.5
    check_int8_rows(W)
    check_int8_rows(W.to(torch.bfloat16))


def check_act(X):
    q, s = wq.quant_act_i8(X.cuda())
    oq, os_, st = oracle.quant_act_i8(*oracle_input(X)[:1], dtype_tag=oracle.BF16)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))


def test_act_quant_w8a8_workload():
    wl = WORKLOADS["w8a8"]
    check_act(wl.activation(4096, 4096))


def test_act_quant_prefill_workload():
    wl = WORKLOADS["prefill"]
    check_act(wl.activation(2048, 4096))


@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (17, 4096), (2, 11008)])
def test_act_quant_ragged(M, K):
    X = make_activation(M, K, seed=M + K, outlier_dims=min(6, K // 8))
    X[0, :] = 0.0
    check_act(X)


# ------------------------------------------- rounding boundaries of the codes
# The quantizers reach fl(x / s) through a reciprocal multiply and decide
# exact half-way quotients (and, for a binary32 scale, quotients within 2^-14
# of a half-way point) separately.  These inputs put most elements on or next
# to those boundaries; codes must still equal the oracle's IEEE-division ones.

def _half_steps(n, step, lo, hi, seed):
    """n values (j + 1/2) * step with integer j in [lo, hi), shuffled."""
    g = torch.Generator().manual_seed(seed)
    j = torch.randint(lo, hi, (n,), generator=g).double()
    return ((j + 0.5) * step).float()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("g", [32, 128, 512])
def test_int4_half_way_quotients(dtype, g):
    rows, K = 12, 2048
    step = 0.0625  # the fp16 scale of every group: amax = 7 step, or range = 15 step
    W = torch.empty(rows, K)
    for r in range(rows):
        W[r] = _half_steps(K, step, -7, 7, seed=r)
    Ws, Wa = W.clone(), W.clone()
    Ws.view(rows, K // g, g)[:, :, 0] = 7 * step          # sym: s = step
    Wa.view(rows, K // g, g)[:, :, 0] = 7 * step
    Wa.view(rows, K // g, g)[:, :, 1] = -8 * step         # asym: s = step, z = 8
    Wa.view(rows, K // g, g)[1::2, :, 1] = -7 * step      # odd rows: range 14 step
    check_int4(Ws.to(dtype), g, sym=True)
    check_int4(Wa.to(dtype), g, sym=False)


def _scale_sweep(rows, K, g, dtype, seed):
    """Groups over a wide range of scales (log-uniform over 2^-22 .. 2^8 of
    the target step, fp16 subnormal scales included), half of them with a
    step of at most 4 significant bits so that (j + 1/2) step is exact in the
    16-bit type (exact half-way quotients), the other half with random
    steps; the elements are j + 1/2 + d steps, d from {0, +-2^-12, +-2^-9,
    uniform(-1/2, 1/2)}, rounded to the type, so quotients crowd around
    rounding points.  Element 0 of each group is 7 steps (sym amax) and
    element 1 is -8 or -7 steps (asym minimum)."""
    rng = np.random.default_rng(seed)
    ng = rows * K // g
    hi_exp = 8 if dtype == torch.bfloat16 else 5
    e = rng.uniform(-22, hi_exp, ng)
    frac = np.where(rng.random(ng) < 0.5, np.round(rng.uniform(8, 16, ng)) / 8,
                    rng.uniform(1, 2, ng))
    step = (frac * np.exp2(np.floor(e))).astype(np.float32).astype(np.float64)
    j = rng.integers(-8, 8, (ng, g)).astype(np.float64)
    d = rng.choice([0.0, 2.0 ** -12, -2.0 ** -12, 2.0 ** -9, -2.0 ** -9, np.nan], (ng, g))
    u = rng.uniform(-0.5, 0.5, (ng, g))
    d = np.where(np.isnan(d), u, d)
    v = (j + 0.5 + d) * step[:, None]
    v[:, 0] = 7 * step
    v[:, 1] = np.where(rng.random(ng) < 0.5, -8, -7) * step
    return torch.from_numpy(v.reshape(rows, K).astype(np.float32)).to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("g", [32, 128, 512])
def test_int4_scale_sweep(dtype, g):
    """Codes follow the IEEE quotient across scales and near every rounding
    point (subnormal fp16 scales take the clamped path)."""
    W = _scale_sweep(256, 4096, g, dtype, seed=g)
    check_int4(W, g, sym=True)
    check_int4(W, g, sym=False)


def _rows_with(X):
    check_int8_rows(X)
    if X.dtype != torch.bfloat16:  # the activation quantizer takes bf16 only
        return
    q, s = wq.quant_act_i8(X.cuda())
    arr, tag = oracle_input(X)
    oq, os_, st = oracle.quant_act_i8(arr, dtype_tag=tag)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("K", [64, 4096, 5120])
def test_int8_rows_half_way(dtype, K):
    """Row maximum 127 2^-7 (scale 2^-7 exactly), values on half-integer
    multiples of the scale."""
    R = 24
    X = torch.stack([_half_steps(K, 2.0 ** -7, -127, 127, seed=r) for r in range(R)])
    X[:, 0] = 127 * 2.0 ** -7
    _rows_with(X.to(dtype))


@pytest.mark.parametrize("K", [64, 4096])
def test_int8_rows_close_to_half_way(K):
    """fp16 rows (maximum 3) whose quotients by the binary32 scale 3/127 lie
    within 2^-9 of a half-integer."""
    s = np.float32(3.0) / np.float32(127.0)
    vals = np.arange(1, 0x4200, dtype=np.uint16).view(np.float16).astype(np.float32)
    vals = vals[vals < 3.0]
    qv = vals / s
    near = vals[np.abs(np.abs(qv - np.rint(qv)) - 0.5) < 2.0 ** -9]
    assert near.size > 8
    rng = np.random.default_rng(K)
    X = rng.choice(near, size=(16, K)) * rng.choice([-1.0, 1.0], size=(16, K))
    X[:, 0] = 3.0
    _rows_with(torch.from_numpy(X.astype(np.float32)).to(torch.float16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fp8_rows_half_way(dtype):
    """amax = 7 gives s = 2^-6; values on E4M3 half-way points (m + 1/2)
    2^(e-3) times s, in the normal and subnormal E4M3 ranges."""
    R, K = 16, 1024
    rng = np.random.default_rng(3)
    e = rng.integers(-9, 8, size=(R, K)).astype(np.float64)
    m = rng.integers(8, 16, size=(R, K)).astype(np.float64)
    v = (m + 0.5) * 2.0 ** (e - 3) * 2.0 ** -6 * rng.choice([-1.0, 1.0], size=(R, K))
    v[:, 0] = 7.0
    A = torch.from_numpy(v.astype(np.float32)).to(dtype)
    q, s = wq.quantize_fp8_rows(A.cuda())
    arr, tag = oracle_input(A)
    oq, os_, st = oracle.quantize_fp8_rows(arr, dtype_tag=tag)
    assert st == oracle.OK
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)


def test_kv_half_way():
    """V rows and K channels whose scale is exactly 2^-7, values on
    half-integer multiples of it."""
    BH, S, D = 2, 64, 128
    Kc = _half_steps(BH * S * D, 2.0 ** -7, -127, 127, seed=1).view(BH, S, D)
    Vc = _half_steps(BH * S * D, 2.0 ** -7, -127, 127, seed=2).view(BH, S, D)
    Kc[:, 0, :] = 127 * 2.0 ** -7
    Vc[:, :, 0] = 127 * 2.0 ** -7
    Kb, Vb = Kc.to(torch.bfloat16), Vc.to(torch.bfloat16)
    qk, sk, qv, sv = wq.quant_kv(Kb.cuda(), Vb.cuda())
    oqk, osk, oqv, osv, st = oracle.quant_kv(bf16_bits(Kb), bf16_bits(Vb), dtype_tag=oracle.BF16)
    assert st == oracle.OK
    np.testing.assert_array_equal(qk.cpu().numpy(), oqk)
    np.testing.assert_array_equal(qv.cpu().numpy(), oqv)
    np.testing.assert_array_equal(sk.cpu().numpy().view(np.uint32), osk.view(np.uint32))
    np.testing.assert_array_equal(sv.cpu().numpy().view(np.uint32), osv.view(np.uint32))


# ------------------------- per-token quantizers with the row held in registers
# 16-bit rows of 1024, 2048, 4096 or 8192 elements go through a kernel that
# reads each row once; its codes and scales must equal the oracle's, like the
# two-pass kernel's (3072 and 5120 take the two-pass kernel).

@pytest.mark.parametrize("M,K", [(1, 1024), (13, 2048), (7, 8192), (3, 3072), (5, 5120)])
def test_act_quant_rows_in_registers(M, K):
    X = make_activation(M, K, seed=M * 7 + K, outlier_dims=6)
    X[-1, :] = 0.0   # an all-zero row takes the 1e-8 floor
    check_act(X)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,K", [(5, 1024), (9, 8192)])
def test_fp8_rows_in_registers(dtype, M, K):
    A = make_activation(M, K, seed=M + 3 * K, outlier_dims=6, dtype=dtype)
    q, s = wq.quantize_fp8_rows(A.cuda())
    arr, tag = oracle_input(A)
    oq, os_, st = oracle.quantize_fp8_rows(arr, dtype_tag=tag)
    assert st == oracle.OK
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)


def test_act_quant_rows_in_registers_non_finite():
    """An infinity counts in the row maximum and a NaN does not, as in the
    oracle; the codes of such rows still match it and the status reports the
    non-finite input."""
    X = make_activation(4, 1024, seed=9).float()
    X[1, 10] = float("inf")
    X[2, 20] = float("nan")
    X = X.to(torch.bfloat16)
    wq.wq_get_device_status(reset=True)
    q, s = wq.quant_act_i8(X.cuda())
    assert wq.wq_get_device_status(reset=True) == wq.WQ_ERR_NONFINITE
    oq, os_, st = oracle.quant_act_i8(bf16_bits(X), dtype_tag=oracle.BF16)
    assert st == oracle.ERR_NONFINITE
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
