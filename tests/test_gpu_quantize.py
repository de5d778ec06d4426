"""GPU parity of the quantize / pack / dequantize / per-row INT8 kernels:
bit-exact against the CPU oracle on the same seeded inputs, at the workloads'
full sizes and on small, ragged and degenerate cases."""
import numpy as np
import pytest
import torch

import bit_gemm_group_b200 as wq
import oracle
from parity_util import oracle_input, u16
from workloads import WORKLOADS, make_weight, make_activation

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
