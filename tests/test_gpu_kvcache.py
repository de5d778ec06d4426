"""GPU parity of the KV-cache INT8 quantizer ("27届大模型面试准备（十九）…"
sec. 6: K per channel, V per token) against the oracle, bit-exact: codes and
scales, for bf16 / fp16 / fp32 caches, ragged token counts and head dims, and
a cache large enough to span many CTA strips per head."""
import numpy as np
import pytest
import torch

import bit_gemm_group_b200 as wq
import oracle
from parity_util import oracle_input

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    wq.wq_get_device_status(reset=True)
    yield
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK


def make_kv(BH, S, D, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    K = torch.randn((BH, S, D), generator=g)
    V = torch.randn((BH, S, D), generator=g)
    if D >= 16:
        K[:, :, [1, D // 3, D - 2]] *= 40.0       # channel-wise outliers in K
    return K.to(dtype), V.to(dtype)


def check(K, V):
    qk, sk, qv, sv = (t.cpu().numpy() for t in wq.quant_kv(K.cuda(), V.cuda()))
    kk, tag = oracle_input(K.reshape(-1, K.shape[-1]))
    vv, _ = oracle_input(V.reshape(-1, V.shape[-1]))
    okq, oks, ovq, ovs, st = oracle.quant_kv(kk.reshape(K.shape), vv.reshape(V.shape), dtype_tag=tag)
    assert st == oracle.OK
    np.testing.assert_array_equal(sk, oks)
    np.testing.assert_array_equal(sv, ovs)
    np.testing.assert_array_equal(qk, okq)
    np.testing.assert_array_equal(qv, ovq)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("BH,S,D", [(1, 1, 8), (3, 37, 64), (2, 300, 128), (5, 17, 256)])
def test_quant_kv_bitexact(dtype, BH, S, D):
    check(*make_kv(BH, S, D, BH * S + D, dtype))


def test_quant_kv_long_heads():
    # 4096 tokens per head: many token strips merge into each channel maximum
    check(*make_kv(16, 4096, 128, 7, torch.bfloat16))


def test_quant_kv_zero_head_clamps_scale():
    K = torch.zeros((2, 64, 128), dtype=torch.bfloat16)
    V = torch.zeros((2, 64, 128), dtype=torch.bfloat16)
    K[1] = 1.0
    check(K, V)
