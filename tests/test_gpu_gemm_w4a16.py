"""GPU parity of the W4A16 prefill product (M > 16, tensor cores) against the
fp64 oracle: max_{m,n} |Y - Y_ref| / ||Y_ref[m, :]||_2 <= 2e-3 (the kernel
multiplies bf16 activations by the bf16-rounded dequantized weight)."""
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


def check(X, dq, oq, sym, windows=None, elementwise=False):
    """Row-normalised bound; with `elementwise`, the bound the arithmetic fixes
    for each output instead: each weight is rounded once to bf16 (relative
    error <= 2^-9), so |Y - Y_ref| <= 2^-8 * sum_k |x_k * w_k| + half a bf16
    ulp of Y (the 2^-8 leaves room for fp32 accumulation)."""
    codes, scales, zeros = dq
    Y = wq.gemm_w4a16(X.cuda(), codes, scales, zeros, 128, sym).float().cpu().numpy()
    N, K = codes.shape[0], X.shape[1]
    for n0, n1 in (windows or [(0, N)]):
        Yref, st = oracle.gemm_w4a16(bf16_bits(X), *oq, 128, sym, n0, n1)
        assert st == oracle.OK
        if elementwise:
            What, _ = oracle.dequant_int4(*oq, K, 128, sym)
            A = np.abs(X.double().numpy()) @ np.abs(What[n0:n1].astype(np.float64)).T
            mag = np.abs(Yref)
            half_ulp = np.where(mag > 0, np.exp2(np.floor(np.log2(np.where(mag > 0, mag, 1))) - 8), 0)
            excess = np.abs(Y[:, n0:n1] - Yref) - (2.0 ** -8 * A + half_ulp)
            assert excess.max() <= 0, (n0, n1, float(excess.max()))
        else:
            err = rel_row_error(Y[:, n0:n1], Yref)
            assert err <= REL_ROW_TOL, (n0, n1, err)
    return Y


def test_prefill_workload_sampled():
    wl = WORKLOADS["prefill"]
    W = wl.weight(0)
    dq, oq = quantized(W, True)
    X = wl.activation(2048, 4096)
    N = W.shape[0]
    # five 256/384-column windows spread over N, at the row-normalised bound
    check(X, dq, oq, True, [(0, 256), (N // 4 - 128, N // 4 + 128), (N // 2 - 128, N // 2 + 128),
                            (3 * N // 4 - 128, 3 * N // 4 + 128), (N - 384, N)])
    check(X[:64], dq, oq, True, [(1000, 1128)], elementwise=True)


@pytest.mark.parametrize("M", [17, 100, 256, 300])
@pytest.mark.parametrize("N,K", [(8, 128), (136, 1152), (264, 4096)])
@pytest.mark.parametrize("sym", [True, False])
def test_ragged(M, N, K, sym):
    W = make_weight(N, K, 0.02, seed=N * 3 + K, outlier_frac=0.01, outlier_scale=30.0)
    dq, oq = quantized(W, sym)
    X = make_activation(M, K, seed=M + 1, outlier_dims=min(6, K // 64))
    check(X, dq, oq, sym, elementwise=True)


def test_matches_dequant_then_matmul():
    """The kernel is X @ dequant_bf16(W)^T with fp32 accumulation."""
    W = make_weight(512, 2048, 0.02, seed=11)
    codes, scales, zeros = wq.quantize_pack(W.cuda(), 128, 4, False)
    X = make_activation(200, 2048, seed=12).cuda()
    Y = wq.gemm_w4a16(X, codes, scales, zeros, 128, False).float()
    Wd = wq.dequant(codes, scales, zeros, 2048, 128, 4, False, torch.bfloat16).float()
    ref = (X.double() @ Wd.double().T)
    A = X.double().abs() @ Wd.double().abs().T
    mag = ref.abs()
    half_ulp = torch.where(mag > 0, torch.exp2(torch.floor(torch.log2(mag.clamp_min(1e-300))) - 8),
                           torch.zeros_like(mag))
    # only the bf16 rounding of Y and fp32 accumulation (~K * 2^-24 relative) separate them
    excess = (Y.double() - ref).abs() - (half_ulp + 2048 * 2.0 ** -24 * A)
    assert excess.max().item() <= 0, excess.max().item()


def test_deterministic():
    W = make_weight(384, 1024, 0.02, seed=5)
    codes, scales, _ = wq.quantize_pack(W.cuda(), 128, 4, True)
    X = make_activation(300, 1024, seed=6).cuda()
    a = wq.gemm_w4a16(X, codes, scales, None)
    b = wq.gemm_w4a16(X, codes, scales, None)
    assert torch.equal(a, b)
