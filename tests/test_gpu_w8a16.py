"""GPU parity of the W8A16 product (int8 or E4M3 per-channel weights, bf16
activations; "27届大模型面试准备（十九）…" sec. 2.3) against the fp64 oracle:
max_{m,n} |Y - Y_ref| / ||Y_ref[m, :]||_2 <= 2e-3.  The weight codes come from
the library's own quantizers (checked bit-exact against the oracle elsewhere)
and are handed to both sides."""
import numpy as np
import pytest
import torch

import bit_gemm_group_b200 as wq
import oracle
from parity_util import REL_ROW_TOL, rel_row_error
from workloads import WORKLOADS, bf16_bits, make_activation, make_weight

pytestmark = pytest.mark.gpu

FORMATS = ["int8", "e4m3"]


@pytest.fixture(autouse=True)
def _clean_status():
    wq.wq_get_device_status(reset=True)
    yield
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK


def weight_codes(W, fmt):
    """(device codes, device scales, oracle format) of a bf16 weight."""
    Wd = W.cuda()
    if fmt == "int8":
        q, s, _ = wq.quantize_pack(Wd, W.shape[1], 8, True)
        return q, s, oracle.W_I8
    q, s = wq.quantize_fp8_rows(Wd)
    return q, s, oracle.W_E4M3


def check(X, q, s, ofmt, windows=None, rounding_aware=False, rows=None):
    Y = wq.gemm_w8a16(X.cuda(), q, s).float().cpu().numpy()
    N = q.shape[0]
    qn, sn = q.cpu().numpy(), s.cpu().numpy()
    Xb = bf16_bits(X)
    if rows is not None:
        Xb, Y = Xb[rows], Y[rows]
    for n0, n1 in windows or [(0, N)]:
        Yref, st = oracle.gemm_w8a16(Xb, qn, ofmt, sn, n0, n1)
        assert st == oracle.OK
        err = rel_row_error(Y[:, n0:n1], Yref, rounding_aware)
        assert err <= REL_ROW_TOL, (n0, n1, err)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("i", [0, 1, 2])
def test_7b_decode_shapes(fmt, i):
    wl = WORKLOADS["7b-decode"]
    W = wl.weight(i)
    q, s, ofmt = weight_codes(W, fmt)
    for M in wl.ms:  # 1 and 4 on the CUDA cores, 16 on the tensor cores
        check(wl.activation(M, W.shape[1]), q, s, ofmt)


@pytest.mark.parametrize("fmt", FORMATS)
def test_prefill_shape_sampled(fmt):
    wl = WORKLOADS["prefill"]
    W = wl.weight(0)
    N, K = W.shape
    q, s, ofmt = weight_codes(W, fmt)
    X = wl.activation(2048, K)
    rows = np.r_[0:8, 1020:1028, 2040:2048]
    windows = [(0, 256), (N // 2 - 128, N // 2 + 128), (N - 256, N)]
    check(X, q, s, ofmt, windows, rows=rows)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 17, 300])
@pytest.mark.parametrize("N,K", [(8, 64), (136, 192), (264, 4160)])
def test_ragged(fmt, M, N, K):
    W = make_weight(N, K, 0.02, seed=N + K, outlier_frac=0.02, outlier_scale=20.0)
    q, s, ofmt = weight_codes(W, fmt)
    X = make_activation(M, K, seed=M + K, outlier_dims=min(6, K // 16))
    check(X, q, s, ofmt, rounding_aware=N < 256)


@pytest.mark.parametrize("fmt", FORMATS)
def test_extreme_codes(fmt):
    """Every code value: int8 -127..127 and all finite E4M3 bytes (subnormals
    included) on the rows of one weight, through both kernels."""
    K = 256
    if fmt == "int8":
        codes = np.arange(-127, 128, dtype=np.int16)
        q = np.resize(codes, (16, K)).astype(np.int8)
        qd = torch.from_numpy(q).cuda()
        ofmt = oracle.W_I8
    else:
        codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
        q = np.resize(codes, (16, K))
        qd = torch.from_numpy(q).cuda()
        ofmt = oracle.W_E4M3
    s = torch.linspace(0.5, 2.0, 16, dtype=torch.float32).cuda()
    for M in (1, 4, 32):
        X = make_activation(M, K, seed=M)
        check(X, qd, s, ofmt, rounding_aware=True)


def test_matches_dequantized_bf16_product():
    """W8A16 with int8 codes equals the bf16 product with the expanded weight
    (every int8 code is exact in bf16) up to accumulation order."""
    W = make_weight(512, 1024, 0.02, seed=9)
    q, s, _ = weight_codes(W, "int8")
    X = make_activation(64, 1024, seed=5).cuda()
    Y = wq.gemm_w8a16(X, q, s).float()
    Wd = q.float() * s[:, None]
    ref = X.double() @ Wd.double().T
    err = ((Y.double() - ref).abs().amax(dim=1) / ref.norm(dim=1)).max().item()
    assert err <= REL_ROW_TOL


def test_non_finite_activation_chunks():
    """int8 codes at M <= 4 read X in fixed point; a chunk of X holding an
    infinity or a NaN is multiplied in fp32 instead, so the row follows IEEE
    arithmetic (inf * 0 = NaN) like the oracle, and the other row stays within
    the tolerance."""
    W = make_weight(64, 1024, 0.02, seed=4)
    q, s, ofmt = weight_codes(W, "int8")
    X = make_activation(3, 1024, seed=8).float()
    X[1, 5] = float("inf")
    X[2, 700] = float("nan")
    X = X.to(torch.bfloat16)
    Y = wq.gemm_w8a16(X.cuda(), q, s).float().cpu().numpy()
    Yref, st = oracle.gemm_w8a16(bf16_bits(X), q.cpu().numpy(), ofmt, s.cpu().numpy(), 0, 64)
    assert np.array_equal(np.isnan(Y[1:]), np.isnan(Yref[1:]))
    assert np.array_equal(np.isinf(Y[1:]), np.isinf(Yref[1:]))
    fin = np.isfinite(Yref[1:])
    assert np.array_equal(np.sign(Y[1:][np.isinf(Y[1:])]), np.sign(Yref[1:][np.isinf(Yref[1:])]))
    assert fin.sum() == 0 or np.all(np.isfinite(Y[1:][fin]))
    err = rel_row_error(Y[:1], Yref[:1], True)
    assert err <= REL_ROW_TOL


def test_arguments():
    X = make_activation(2, 128, seed=1).cuda()
    q = torch.zeros((16, 128), dtype=torch.int8, device="cuda")
    s = torch.ones(16, dtype=torch.float32, device="cuda")
    Y = torch.empty((2, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w8a16(X, q, 7, s, Y)
    assert e.value.status == wq.WQ_ERR_ARG
    X2 = make_activation(2, 96, seed=1).cuda()
    q2 = torch.zeros((16, 96), dtype=torch.int8, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w8a16(X2, q2, wq.WQ_W8_INT8, s, Y)
    assert e.value.status == wq.WQ_ERR_ALIGN
