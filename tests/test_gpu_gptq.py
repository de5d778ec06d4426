"""GPU parity of GPTQ ("27届大模型面试准备（十九）…" sec. 4.3) against the oracle:
codes, scales and zeros equal (both sides correct in binary64 and decide in
binary32; only the order of the binary64 sums differs), an identity factor
reproduces the round-to-nearest quantizer, and GPTQ lowers the layer's
reconstruction error on correlated calibration data."""
import numpy as np
import pytest
import torch

import bit_gemm_group_b200 as wq
import oracle
from parity_util import oracle_input
from workloads import make_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    wq.wq_get_device_status(reset=True)
    yield
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK


def calib(T, K, seed):
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((T, K // 8))
    return (base @ rng.standard_normal((K // 8, K)) + 0.2 * rng.standard_normal((T, K))).astype(np.float32)


def u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("N,K,dtype", [(1, 128, torch.float32), (37, 384, torch.bfloat16),
                                       (256, 1024, torch.bfloat16), (70, 512, torch.float16)])
def test_gptq_matches_oracle(N, K, dtype, sym):
    X = calib(2 * K, K, seed=K + N)
    U, st = oracle.gptq_hinv_chol(X, 0.01)
    assert st == oracle.OK
    W = make_weight(N, K, 0.02, seed=N + K, outlier_frac=0.01, outlier_scale=20.0, dtype=dtype)
    c, s, z = wq.gptq_quantize(W.cuda(), torch.from_numpy(U).cuda(), sym)
    arr, tag = oracle_input(W)
    oc, osc, oz, st = oracle.gptq_quantize(arr, U, 128, sym, dtype_tag=tag)
    assert st == oracle.OK
    np.testing.assert_array_equal(u16(s), osc)
    if not sym:
        np.testing.assert_array_equal(u16(z), oz)
    np.testing.assert_array_equal(c.cpu().numpy(), oc)


@pytest.mark.parametrize("sym", [True, False])
def test_identity_factor_is_round_to_nearest(sym):
    W = make_weight(300, 1024, 0.02, seed=5).cuda()
    c, s, z = wq.gptq_quantize(W, torch.eye(1024, dtype=torch.float64, device="cuda"), sym)
    rc, rs, rz = wq.quantize_pack(W, 128, 4, sym)
    assert torch.equal(c, rc) and torch.equal(s, rs)
    if not sym:
        assert torch.equal(z, rz)


def test_gptq_lowers_reconstruction_error_on_gpu():
    K = 1024
    X = calib(2048, K, seed=9)
    U, _ = oracle.gptq_hinv_chol(X, 0.01)
    W = make_weight(512, K, 0.02, seed=9).cuda()
    g = wq.gptq_quantize(W, torch.from_numpy(U).cuda(), True)
    r = wq.quantize_pack(W, 128, 4, True)

    def err(q):
        What = torch.empty((512, K), dtype=torch.float32, device="cuda")
        wq.wq_dequant(q[0], q[1], q[2], 512, K, 128, 4, True, What)
        d = torch.from_numpy(X).double() @ (W.double().cpu() - What.double().cpu()).T
        return float(d.norm())

    assert err(g) < 0.8 * err(r)
