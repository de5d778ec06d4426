"""GPU parity of the W4A16 decode product (M <= 16) against the fp64 oracle:
max_{m,n} |Y - Y_ref| / ||Y_ref[m, :]||_2 <= 2e-3, on the workloads' full
shapes (sampled output columns for the 70B shapes) and on ragged cases."""
import numpy as np
import pytest
import torch

import bit_gemm_group_b200 as wq
import oracle
from parity_util import REL_ROW_TOL, oracle_input, rel_row_error
from workloads import WORKLOADS, make_activation, make_weight, bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    wq.wq_get_device_status(reset=True)
    yield
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK


def quantized(W, sym):
    codes, scales, zeros = wq.quantize_pack(W.cuda(), 128, 4, sym)
    arr, tag = oracle_input(W)
    oc, osc, oz, _ = oracle.quantize_int4(arr, 128, sym, dtype_tag=tag)
    return (codes, scales, zeros), (oc, osc, oz)


def check_gemv(X, dev_q, ora_q, sym, windows=None, rounding_aware=False):
    codes, scales, zeros = dev_q
    Y = wq.gemm_w4a16(X.cuda(), codes, scales, zeros, 128, sym).float().cpu().numpy()
    N = codes.shape[0]
    windows = windows or [(0, N)]
    for n0, n1 in windows:
        Yref, st = oracle.gemm_w4a16(bf16_bits(X), *ora_q, 128, sym, n0, n1)
        assert st == oracle.OK
        err = rel_row_error(Y[:, n0:n1], Yref, rounding_aware)
        assert err <= REL_ROW_TOL, (n0, n1, err)
    return Y


def test_tiny_workload():
    wl = WORKLOADS["tiny"]
    W = wl.weight(0)
    dq, oq = quantized(W, wl.sym)
    check_gemv(wl.activation(1, 512), dq, oq, wl.sym)


@pytest.mark.parametrize("i", [0, 1, 2])
def test_7b_decode_full(i):
    wl = WORKLOADS["7b-decode"]
    W = wl.weight(i)
    dq, oq = quantized(W, True)
    for M in wl.ms:
        check_gemv(wl.activation(M, W.shape[1]), dq, oq, True)


@pytest.mark.parametrize("i", [0, 1])
def test_70b_decode_sampled(i):
    wl = WORKLOADS["70b-decode"]
    W = wl.weight(i)
    N = W.shape[0]
    dq, oq = quantized(W, False)
    windows = [(0, 256), (N // 2 - 128, N // 2 + 128), (N - 256, N)]
    for M in wl.ms:
        check_gemv(wl.activation(M, W.shape[1]), dq, oq, False, windows)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 13, 16])
@pytest.mark.parametrize("N,K", [(8, 128), (24, 256), (136, 1152), (264, 4096)])
@pytest.mark.parametrize("sym", [True, False])
def test_ragged(M, N, K, sym):
    W = make_weight(N, K, 0.02, seed=N + K, outlier_frac=0.01, outlier_scale=30.0)
    dq, oq = quantized(W, sym)
    check_gemv(make_activation(M, K, seed=M), dq, oq, sym, rounding_aware=N < 256)


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("N,K", [(8, 1152), (24, 1152), (136, 4096)])
@pytest.mark.parametrize("sym", [True, False])
def test_small_n_with_outlier_activations(M, N, K, sym):
    """Few outputs per row and six activation dims of magnitude 50-100: the
    CUDA-core kernel rounds each group's activations to 13-bit integers
    relative to the group maximum, so a group that holds an outlier dim
    rounds nearly all its other elements; with small N one output carries
    much of the row norm.  The row-normalised bound (less the bf16 output
    half-ulp) still holds."""
    W = make_weight(N, K, 0.02, seed=N + 7 * K, outlier_frac=0.01, outlier_scale=30.0)
    dq, oq = quantized(W, sym)
    X = make_activation(M, K, seed=M + 31, outlier_dims=6)
    check_gemv(X, dq, oq, sym, rounding_aware=True)


@pytest.mark.parametrize("kind", ["positive", "outlier_dims", "row_scales", "sparse_groups"])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_activation_structure(kind, M):
    """Activation value structure that stresses the per-(group, row) handling:
    all-positive values (large same-sign sums), outlier hidden dims of
    magnitude 50-100, rows whose magnitudes differ by 10^6, and groups that
    are entirely zero."""
    N, K = 4096, 4096
    W = make_weight(N, K, 0.02, seed=11, outlier_frac=0.001, outlier_scale=30.0)
    dq, oq = quantized(W, False)
    if kind == "outlier_dims":
        X = make_activation(M, K, seed=M, outlier_dims=6)
    else:
        X = make_activation(M, K, seed=M).float()
        if kind == "positive":
            X = X.abs() + 0.5
        elif kind == "row_scales":
            X = X * torch.logspace(-3, 3, M).reshape(M, 1) if M > 1 else X * 1e-3
        else:
            X.view(M, K // 128, 128)[:, 1::3, :] = 0.0
        X = X.to(torch.bfloat16)
    check_gemv(X, dq, oq, False)


def test_workspace_reused_and_left_zeroed():
    W = make_weight(1000 * 8, 4096, 0.02, seed=3)
    dq, oq = quantized(W, True)
    codes, scales, zeros = dq
    X = make_activation(2, 4096, seed=4).cuda()
    ws = wq.w4a16_workspace(2, W.shape[0], 4096, "cuda")
    outs = [wq.gemm_w4a16(X, codes, scales, zeros, ws=ws) for _ in range(3)]
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    T = (W.shape[0] + 127) // 128
    assert int(ws[: 4 * T].count_nonzero()) == 0  # arrival counters reset by every call


def test_workspace_shared_by_both_decode_kernels():
    """One workspace serves the CUDA-core kernel (M <= 4) and the tensor-core
    kernel (M = 5..16) alternately."""
    N, K = 4096, 4096
    W = make_weight(N, K, 0.02, seed=5)
    (codes, scales, zeros), _ = quantized(W, False)
    Xs = {M: make_activation(M, K, seed=M).cuda() for M in (1, 2, 4, 8, 16)}
    ref = {M: wq.gemm_w4a16(X, codes, scales, zeros, 128, False) for M, X in Xs.items()}
    nbytes = max(wq.lib().wq_w4a16_workspace_bytes(M, N, K) for M in Xs)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for M in (1, 8, 2, 16, 1, 4, 8):
        Y = wq.gemm_w4a16(Xs[M], codes, scales, zeros, 128, False, ws=ws)
        assert torch.equal(Y, ref[M]), M
    assert int(ws[: 4 * (N // 128)].count_nonzero()) == 0


def test_workspace_too_small():
    W = make_weight(256, 1024, 0.02, seed=3).cuda()
    codes, scales, _ = wq.quantize_pack(W, 128, 4, True)
    X = make_activation(1, 1024, seed=4).cuda()
    Y = torch.empty(1, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w4a16(X, codes, scales, None, 256, 128, True, Y, None)
    assert e.value.status == wq.WQ_ERR_WORKSPACE


@pytest.mark.parametrize("M", [1, 2, 4])
def test_deterministic(M):
    wl = WORKLOADS["7b-decode"]
    W = wl.weight(1)
    (codes, scales, zeros), _ = quantized(W, True)
    X = wl.activation(M, W.shape[1]).cuda()
    a = wq.gemm_w4a16(X, codes, scales, zeros)
    b = wq.gemm_w4a16(X, codes, scales, zeros)
    assert torch.equal(a, b)
