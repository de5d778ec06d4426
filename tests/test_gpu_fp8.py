"""GPU parity of the FP8 E4M3 W8A8 path against the oracle: E4M3 codes and
scales bit-exact, the tensor cores' fp32 accumulators within the rounding of
an fp32 sum of exact products, and Y within 2e-3 (row-normalised)."""
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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32, torch.float16])
@pytest.mark.parametrize("R,K", [(1, 16), (37, 1040), (4096, 4096)])
def test_quantize_fp8_rows_bitexact(dtype, R, K):
    A = make_activation(R, K, seed=R + K, outlier_dims=min(6, K // 16), dtype=dtype)
    q, s = wq.quantize_fp8_rows(A.cuda())
    oq, os_, st = oracle.quantize_fp8_rows(*oracle_input(A)[:1], dtype_tag=oracle_input(A)[1])
    assert st == oracle.OK
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)


def run_case(W, X, windows):
    qw, sw = wq.quantize_fp8_rows(W.cuda())
    Y, acc = wq.gemm_fp8(X.cuda(), qw, sw, want_acc=True)
    Y, acc = Y.float().cpu().numpy(), acc.cpu().numpy().astype(np.float64)
    oqw, osw, _ = oracle.quantize_fp8_rows(*oracle_input(W)[:1], dtype_tag=oracle_input(W)[1])
    oqx, osx, _ = oracle.quantize_fp8_rows(bf16_bits(X), dtype_tag=oracle.BF16)
    vx = oracle.e4m3_to_f32(np.arange(256, dtype=np.uint8)).astype(np.float64)
    for m0, m1, n0, n1 in windows:
        Yref, exact, st = oracle.gemm_fp8(oqx, osx, oqw, osw, m0, m1, n0, n1)
        assert st == oracle.OK
        # fp32 accumulation of exact products: within K * 2^-23 of sum |p|
        absum = np.abs(vx[oqx[m0:m1]]) @ np.abs(vx[oqw[n0:n1]]).T
        K = X.shape[1]
        assert np.all(np.abs(acc[m0:m1, n0:n1] - exact) <= K * 2.0 ** -23 * absum + 1e-30)
        err = rel_row_error(Y[m0:m1, n0:n1], Yref, (n1 - n0) < 256)
        assert err <= REL_ROW_TOL, (m0, n0, err)


def test_gemm_fp8_workload_sampled():
    wl = WORKLOADS["w8a8"]
    run_case(wl.weight(0), wl.activation(4096, 4096),
             [(0, 128, 0, 256), (1920, 2176, 1000, 1512), (3968, 4096, 3840, 4096)])


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (129, 272, 256), (200, 512, 1040)])
def test_gemm_fp8_ragged(M, N, K):
    W = make_weight(N, K, 0.02, seed=N + K)
    X = make_activation(M, K, seed=M + K, outlier_dims=min(6, K // 16))
    run_case(W, X, [(0, M, 0, N)])


def test_fp8_more_accurate_than_int8_on_gpu():
    W = make_weight(1024, 2048, 0.02, seed=31, outlier_frac=0.001, outlier_scale=30.0)
    X = make_activation(512, 2048, seed=32, outlier_dims=6)
    Wc, Xc = W.cuda(), X.cuda()
    Yref = X.double().numpy() @ W.double().numpy().T
    qw, sw, _ = wq.quantize_pack(Wc, 2048, 8, True)
    e8 = np.linalg.norm(wq.gemm_w8a8(Xc, qw, sw).double().cpu().numpy() - Yref)
    fw, fsw = wq.quantize_fp8_rows(Wc)
    ef = np.linalg.norm(wq.gemm_fp8(Xc, fw, fsw).double().cpu().numpy() - Yref)
    assert ef < 0.75 * e8, (e8 / np.linalg.norm(Yref), ef / np.linalg.norm(Yref))
