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


@pytest.mark.parametrize("BH,S,D", [(2, 16384, 128), (1, 20000, 64), (3, 2049, 256), (4, 1000, 16)])
def test_quant_kv_token_counts(BH, S, D):
    # cluster sizes 1..8, every channel block width, and S beyond the
    # one-launch kernel's reach (the multi-kernel path)
    check(*make_kv(BH, S, D, S + D, torch.bfloat16))


def test_quant_kv_full_cache():
    """The bench's cache: 8 kv heads x 8 sequences, 8192 tokens, head dim 128."""
    check(*make_kv(64, 8192, 128, 11, torch.bfloat16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_quant_kv_non_finite(dtype):
    """An infinity counts in a maximum and a NaN does not (the oracle's
    comparison), codes of NaN and of an infinity over an infinite scale are
    127, and the status reports the non-finite input."""
    K, V = make_kv(3, 700, 64, 5, torch.float32)
    K[0, 10, 3] = float("inf")
    K[1, 20, 7] = float("nan")
    K[2, 30, 9] = float("-inf")
    K[2, 31, 9] = float("nan")
    V[0, 5, 1] = float("nan")
    V[1, 6, 2] = float("-inf")
    V[2, 7, 3] = float("inf")
    V[2, 7, 4] = float("nan")
    K, V = K.to(dtype), V.to(dtype)
    qk, sk, qv, sv = (t.cpu().numpy() for t in wq.quant_kv(K.cuda(), V.cuda()))
    assert wq.wq_get_device_status(reset=True) == wq.WQ_ERR_NONFINITE
    kk, tag = oracle_input(K.reshape(-1, K.shape[-1]))
    vv, _ = oracle_input(V.reshape(-1, V.shape[-1]))
    okq, oks, ovq, ovs, st = oracle.quant_kv(kk.reshape(K.shape), vv.reshape(V.shape), dtype_tag=tag)
    assert st == oracle.ERR_NONFINITE
    np.testing.assert_array_equal(sk.view(np.uint32), oks.view(np.uint32))
    np.testing.assert_array_equal(sv.view(np.uint32), ovs.view(np.uint32))
    np.testing.assert_array_equal(qk, okq)
    np.testing.assert_array_equal(qv, ovq)


def test_quant_kv_zero_head_clamps_scale():
    K = torch.zeros((2, 64, 128), dtype=torch.bfloat16)
    V = torch.zeros((2, 64, 128), dtype=torch.bfloat16)
    K[1] = 1.0
    check(K, V)
