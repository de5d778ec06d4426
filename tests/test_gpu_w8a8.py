"""GPU parity of the W8A8 product: int32 accumulators bit-exact against the
oracle's exact integer sums (oracle-quantized activations and weights), and
the bf16 output within 2e-3 of the fp64 rescale (row-normalised)."""
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


def run_case(W, X, windows=None, rounding_aware=False):
    N, K = W.shape
    M = X.shape[0]
    qw, sw, _ = wq.quantize_pack(W.cuda(), K, 8, True)
    Y, acc = wq.gemm_w8a8(X.cuda(), qw, sw, want_acc=True)
    Y = Y.float().cpu().numpy()
    acc = acc.cpu().numpy()
    oqw, osw, _ = oracle.quantize_int8_rows(*oracle_input(W)[:1], dtype_tag=oracle_input(W)[1])
    oqx, osx, _ = oracle.quant_act_i8(bf16_bits(X), dtype_tag=oracle.BF16)
    windows = windows or [(0, M, 0, N)]
    for m0, m1, n0, n1 in windows:
        ref_acc, st = oracle.gemm_w8a8_acc(oqx, oqw, m0, m1, n0, n1)
        assert st == oracle.OK
        np.testing.assert_array_equal(acc[m0:m1, n0:n1], ref_acc)
        Yref, _ = oracle.w8a8_rescale(ref_acc, osx, osw, m0, n0)
        err = rel_row_error(Y[m0:m1, n0:n1], Yref, rounding_aware or (n1 - n0) < 256)
        assert err <= REL_ROW_TOL, (m0, n0, err)


def test_w8a8_workload_sampled():
    wl = WORKLOADS["w8a8"]
    W = wl.weight(0)
    X = wl.activation(4096, 4096)
    run_case(W, X, [(0, 128, 0, 256), (1920, 2176, 1000, 1512), (3968, 4096, 3840, 4096),
                    (0, 4096, 2048, 2064)])


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (3, 48, 144), (129, 272, 256),
                                   (300, 512, 4096), (128, 256, 128), (200, 4096, 1040)])
def test_w8a8_ragged(M, N, K):
    W = make_weight(N, K, 0.02, seed=N + K)
    X = make_activation(M, K, seed=M + K, outlier_dims=min(6, K // 16))
    run_case(W, X, rounding_aware=N < 256)


def test_w8a8_deterministic():
    W = make_weight(512, 1024, 0.02, seed=1)
    X = make_activation(256, 1024, seed=2, outlier_dims=6)
    qw, sw, _ = wq.quantize_pack(W.cuda(), 1024, 8, True)
    a = wq.gemm_w8a8(X.cuda(), qw, sw)
    b = wq.gemm_w8a8(X.cuda(), qw, sw)
    assert torch.equal(a, b)


def test_w8a8_workspace_too_small():
    W = make_weight(64, 256, 0.02, seed=1).cuda()
    X = make_activation(32, 256, seed=2).cuda()
    qw, sw, _ = wq.quantize_pack(W, 256, 8, True)
    Y = torch.empty(32, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w8a8(X, qw, sw, Y, ws)
    assert e.value.status == wq.WQ_ERR_WORKSPACE
