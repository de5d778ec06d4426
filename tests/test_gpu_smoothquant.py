"""GPU parity of SmoothQuant smoothing ("27届大模型面试准备（十九）…" sec. 4.2)
against the oracle: the channel statistics bit-exact, the migration factors
within one fp32 ulp (both sides evaluate pow in binary64), the smoothed INT8
weights and activations bit-exact given the oracle's factors, the W8A8
accumulators bit-exact and Y within 2e-3 (row-normalised); and the page's
point that smoothing makes W8A8 on outlier activations more accurate."""
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


def oracle_scales(X, W, alpha=0.5):
    a, _ = oracle.channel_absmax(*oracle_input(X)[:1], dtype_tag=oracle_input(X)[1])
    w, _ = oracle.channel_absmax(*oracle_input(W)[:1], dtype_tag=oracle_input(W)[1])
    s, st = oracle.smooth_scales(a, w, alpha)
    assert st == oracle.OK
    return a, w, s


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32, torch.float16])
@pytest.mark.parametrize("R,K", [(1, 8), (3, 24), (257, 1040), (4096, 4096)])
def test_channel_absmax_bitexact(dtype, R, K):
    A = make_activation(R, K, seed=R + K, outlier_dims=min(6, K // 8), dtype=dtype)
    got = wq.channel_absmax(A.cuda()).cpu().numpy()
    ref, st = oracle.channel_absmax(*oracle_input(A)[:1], dtype_tag=oracle_input(A)[1])
    assert st == oracle.OK
    np.testing.assert_array_equal(got, ref)


def test_channel_absmax_weight_columns():
    W = WORKLOADS["w8a8"].weight(0)
    got = wq.channel_absmax(W.cuda()).cpu().numpy()
    ref, _ = oracle.channel_absmax(*oracle_input(W)[:1], dtype_tag=oracle_input(W)[1])
    np.testing.assert_array_equal(got, ref)


def test_channel_absmax_reports_non_finite():
    A = make_activation(64, 64, seed=1, dtype=torch.float32)
    A[5, 3] = float("inf")
    got = wq.channel_absmax(A.cuda()).cpu().numpy()
    assert wq.wq_get_device_status(reset=True) == wq.WQ_ERR_NONFINITE
    ref, st = oracle.channel_absmax(A.numpy())
    assert st == oracle.ERR_NONFINITE
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.8, 1.0])
def test_smooth_scales_within_one_ulp(alpha):
    rng = np.random.default_rng(7)
    a = np.exp(rng.normal(0, 2, 4096)).astype(np.float32)
    w = np.exp(rng.normal(-4, 1, 4096)).astype(np.float32)
    a[:3] = [0.0, 5.0, 1e-30]
    w[:3] = [0.3, 0.0, 1e-7]
    alpha = float(np.float32(alpha))  # the C ABI takes alpha as fp32; both sides use that value
    s = wq.smooth_scales(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda(), alpha)
    s = s.cpu().numpy()
    ref, _ = oracle.smooth_scales(a, w, alpha)
    ulp = np.spacing(np.abs(ref))
    assert np.all(np.abs(s - ref) <= ulp), np.max(np.abs(s - ref) / ulp)


@pytest.mark.parametrize("N,K", [(16, 48), (300, 1040), (4096, 4096)])
def test_quantize_i8_smooth_bitexact(N, K):
    W = make_weight(N, K, 0.02, seed=N, outlier_frac=0.001, outlier_scale=30.0)
    X = make_activation(64, K, seed=K, outlier_dims=6)
    _, _, s = oracle_scales(X, W)
    q, sc = wq.quantize_i8_smooth(W.cuda(), torch.from_numpy(s).cuda())
    oq, osc, st = oracle.quantize_int8_rows_smoothed(*oracle_input(W)[:1], s,
                                                      dtype_tag=oracle_input(W)[1])
    assert st == oracle.OK
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(sc.cpu().numpy(), osc)


@pytest.mark.parametrize("M,K", [(1, 16), (37, 1040), (4096, 4096)])
def test_quant_act_i8_smooth_bitexact(M, K):
    X = make_activation(M, K, seed=M + 3, outlier_dims=min(6, K // 8))
    W = make_weight(128, K, 0.02, seed=K + 1)
    _, _, s = oracle_scales(X, W)
    q, sx = wq.quant_act_i8_smooth(X.cuda(), torch.from_numpy(s).cuda())
    oq, osx, st = oracle.quant_act_i8_smoothed(bf16_bits(X), s, dtype_tag=oracle.BF16)
    assert st == oracle.OK
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(sx.cpu().numpy(), osx)


def run_smoothed(W, X, windows):
    N, K = W.shape
    M = X.shape[0]
    _, _, s = oracle_scales(X, W)
    st_ = torch.from_numpy(s).cuda()
    qw, sw = wq.quantize_i8_smooth(W.cuda(), st_)
    Y, acc = wq.gemm_w8a8_smooth(X.cuda(), qw, sw, st_, want_acc=True)
    Y, acc = Y.float().cpu().numpy(), acc.cpu().numpy()
    oqw, osw, _ = oracle.quantize_int8_rows_smoothed(*oracle_input(W)[:1], s,
                                                     dtype_tag=oracle_input(W)[1])
    oqx, osx, _ = oracle.quant_act_i8_smoothed(bf16_bits(X), s, dtype_tag=oracle.BF16)
    for m0, m1, n0, n1 in windows:
        ref_acc, st = oracle.gemm_w8a8_acc(oqx, oqw, m0, m1, n0, n1)
        assert st == oracle.OK
        np.testing.assert_array_equal(acc[m0:m1, n0:n1], ref_acc)
        Yref, _ = oracle.w8a8_rescale(ref_acc, osx, osw, m0, n0)
        err = rel_row_error(Y[m0:m1, n0:n1], Yref, (n1 - n0) < 256)
        assert err <= REL_ROW_TOL, (m0, n0, err)


def test_gemm_w8a8_smooth_workload_sampled():
    wl = WORKLOADS["w8a8"]
    run_smoothed(wl.weight(0), wl.activation(4096, 4096),
                 [(0, 128, 0, 256), (1920, 2176, 1000, 1512), (3968, 4096, 3840, 4096)])


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (129, 272, 256), (200, 512, 1040)])
def test_gemm_w8a8_smooth_ragged(M, N, K):
    W = make_weight(N, K, 0.02, seed=N + K)
    X = make_activation(M, K, seed=M + K, outlier_dims=min(6, K // 16))
    run_smoothed(W, X, [(0, M, 0, N)])


def test_smoothing_improves_w8a8_on_outlier_activations():
    """End to end on the GPU: statistics, factors, smoothed quantization and the
    product, against the unquantized fp64 product of the same bf16 inputs."""
    W = make_weight(1024, 2048, 0.02, seed=21)
    X = make_activation(512, 2048, seed=22, outlier_dims=6)
    Wc, Xc = W.cuda(), X.cuda()
    Yref = X.double().numpy() @ W.double().numpy().T
    qw, sw, _ = wq.quantize_pack(Wc, 2048, 8, True)
    e_plain = np.linalg.norm(wq.gemm_w8a8(Xc, qw, sw).double().cpu().numpy() - Yref)
    s = wq.smooth_scales(wq.channel_absmax(Xc), wq.channel_absmax(Wc), 0.5)
    qws, sws = wq.quantize_i8_smooth(Wc, s)
    e_smooth = np.linalg.norm(wq.gemm_w8a8_smooth(Xc, qws, sws, s).double().cpu().numpy() - Yref)
    assert e_smooth < 0.5 * e_plain, (e_plain / np.linalg.norm(Yref), e_smooth / np.linalg.norm(Yref))
