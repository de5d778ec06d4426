"""The C-ABI library loads, exports every symbol include/wq.h declares, and
rejects bad arguments on the host (no GPU needed: validation returns before
any CUDA call; no compute call is made here)."""
import ctypes
import os
import re

import pytest
import torch

import bit_gemm_group_b200 as wq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    wq.build()
    return wq.lib()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "wq.h")).read()
    return sorted(set(re.findall(r"WQ_API\s+[\w\s\*]*?\b(wq_\w+)\s*\(", text)))


def test_header_declares_the_python_list():
    assert _declared_symbols() == sorted(wq.EXPORTED)


def test_every_declared_symbol_is_exported(L):
    for name in _declared_symbols():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in [(0, "WQ_OK"), (-1, "WQ_ERR_ARG"), (-2, "WQ_ERR_UNSUPPORTED"),
                       (-3, "WQ_ERR_ALIGN"), (-6, "WQ_ERR_TIMEOUT"), (-9, "WQ_ERR_NO_DEVICE")]:
        assert wq.wq_status_str(code) == name


def test_workspace_size(L):
    assert wq.wq_w8a8_workspace_bytes(4096, 4096) == 4096 * 4096 + 4096 * 4
    assert wq.wq_w8a8_workspace_bytes(3, 128) == 512 + 256
    assert wq.wq_w8a8_workspace_bytes(0, 128) == 0


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def test_quantize_validation(L):
    q = L.wq_quantize_pack
    assert q(FAKE, 1, -1, 128, 128, 4, 1, FAKE, FAKE, None, None) == wq.WQ_ERR_ARG
    assert q(FAKE, 1, 8, 200, 128, 4, 1, FAKE, FAKE, None, None) == wq.WQ_ERR_ARG      # K % g
    assert q(FAKE, 1, 8, 256, 128, 4, 1, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_ARG      # sym with zeros
    assert q(FAKE, 1, 8, 256, 128, 4, 0, FAKE, FAKE, None, None) == wq.WQ_ERR_ARG      # asym w/o zeros
    assert q(FAKE, 1, 8, 240, 48, 4, 1, FAKE, FAKE, None, None) == wq.WQ_ERR_UNSUPPORTED
    assert q(FAKE, 1, 8, 256, 128, 3, 1, FAKE, FAKE, None, None) == wq.WQ_ERR_UNSUPPORTED
    assert q(FAKE, 7, 8, 256, 128, 4, 1, FAKE, FAKE, None, None) == wq.WQ_ERR_ARG      # dtype
    assert q(MISALIGNED, 1, 8, 256, 128, 4, 1, FAKE, FAKE, None, None) == wq.WQ_ERR_ALIGN
    assert q(FAKE, 1, 8, 256, 256, 8, 0, FAKE, FAKE, None, None) == wq.WQ_ERR_ARG      # int8 asym
    assert q(FAKE, 1, 8, 256, 128, 8, 1, FAKE, FAKE, None, None) == wq.WQ_ERR_ARG      # int8 g != K
    assert q(None, 1, 0, 256, 128, 4, 1, None, None, None, None) == wq.WQ_OK          # empty


def test_dequant_validation(L):
    d = L.wq_dequant
    assert d(FAKE, FAKE, None, 8, 256, 128, 4, 1, FAKE, 2, None) == wq.WQ_ERR_ARG       # fp16 out
    assert d(FAKE, FAKE, FAKE, 8, 256, 128, 4, 1, FAKE, 0, None) == wq.WQ_ERR_ARG
    assert d(FAKE, FAKE, None, 0, 256, 128, 4, 1, FAKE, 0, None) == wq.WQ_OK


def test_gemm_w4a16_validation(L):
    g = L.wq_gemm_w4a16
    assert g(FAKE, 1, 4096, FAKE, FAKE, None, 4096, 64, 1, FAKE, FAKE, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert g(FAKE, 1, 4000, FAKE, FAKE, None, 4096, 128, 1, FAKE, FAKE, 1 << 20, None) == wq.WQ_ERR_ALIGN
    assert g(FAKE, 1, 4096, FAKE, FAKE, None, 4100, 128, 1, FAKE, FAKE, 1 << 20, None) == wq.WQ_ERR_ALIGN
    assert g(FAKE, 1, 4096, FAKE, FAKE, FAKE, 4096, 128, 1, FAKE, FAKE, 1 << 20, None) == wq.WQ_ERR_ARG
    assert g(FAKE, 0, 4096, FAKE, FAKE, None, 4096, 128, 1, FAKE, None, 0, None) == wq.WQ_OK
    assert g(MISALIGNED, 1, 4096, FAKE, FAKE, None, 4096, 128, 1, FAKE, FAKE, 1 << 20, None) == wq.WQ_ERR_ALIGN
    assert g(FAKE, 1, 4096, FAKE, FAKE, None, 4096, 128, 1, FAKE, MISALIGNED, 1 << 20, None) == wq.WQ_ERR_ALIGN


def test_act_quant_validation(L):
    a = L.wq_quant_act_i8
    assert a(FAKE, 4, 100, FAKE, FAKE, None) == wq.WQ_ERR_ALIGN
    assert a(FAKE, -4, 128, FAKE, FAKE, None) == wq.WQ_ERR_ARG
    assert a(FAKE, 0, 128, FAKE, FAKE, None) == wq.WQ_OK


def test_binding_refuses_cpu_tensors(L):
    import torch
    W = torch.zeros(8, 256)
    with pytest.raises(wq.WQError):
        wq.quantize_pack(W)


def test_oracle_builds():
    import oracle
    assert os.path.exists(oracle.build.build())


def test_smoothquant_validation(L):
    # host-side checks return before any device work
    assert L.wq_channel_absmax(FAKE, 1, 8, 12, FAKE, None) == wq.WQ_ERR_ALIGN          # K % 8
    assert L.wq_channel_absmax(FAKE, 9, 8, 16, FAKE, None) == wq.WQ_ERR_ARG            # dtype
    assert L.wq_channel_absmax(MISALIGNED, 1, 8, 16, FAKE, None) == wq.WQ_ERR_ALIGN
    assert L.wq_channel_absmax(FAKE, 1, 8, 0, FAKE, None) == wq.WQ_OK
    assert L.wq_smooth_scales(FAKE, FAKE, 16, 1.5, FAKE, None) == wq.WQ_ERR_ARG        # alpha
    assert L.wq_smooth_scales(FAKE, FAKE, 16, -0.1, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_smooth_scales(None, FAKE, 16, 0.5, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_quantize_i8_smooth(FAKE, 1, 8, 24, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_ALIGN
    assert L.wq_quantize_i8_smooth(FAKE, 1, 8, 32, None, FAKE, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_quant_act_i8_smooth(FAKE, 8, 32, None, FAKE, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_quant_act_i8_smooth(FAKE, 8, 40, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_ALIGN
    assert L.wq_gemm_w8a8_smooth(FAKE, 8, 128, FAKE, FAKE, None, 16, FAKE, FAKE, 1 << 20,
                                 None, None) == wq.WQ_ERR_ARG
    assert L.wq_gemm_w8a8_smooth(FAKE, 8, 128, FAKE, FAKE, FAKE, 16, FAKE, FAKE, 0,
                                 None, None) == wq.WQ_ERR_WORKSPACE


def test_quant_kv_validation(L):
    assert L.wq_quant_kv(FAKE, FAKE, 1, 2, 8, 12, FAKE, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_ALIGN
    assert L.wq_quant_kv(FAKE, FAKE, 1, 2, 8, 264, FAKE, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_quant_kv(FAKE, FAKE, 5, 2, 8, 128, FAKE, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_quant_kv(FAKE, None, 1, 2, 8, 128, FAKE, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_quant_kv(FAKE, FAKE, 1, 70000, 8, 128, FAKE, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_quant_kv(FAKE, FAKE, 1, 0, 8, 128, FAKE, FAKE, FAKE, FAKE, None) == wq.WQ_OK


def test_fp8_validation(L):
    assert L.wq_quantize_fp8_rows(FAKE, 1, 8, 24, FAKE, FAKE, None) == wq.WQ_ERR_ALIGN
    assert L.wq_quantize_fp8_rows(FAKE, 4, 8, 32, FAKE, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_quantize_fp8_rows(FAKE, 1, 0, 32, FAKE, FAKE, None) == wq.WQ_OK
    assert L.wq_gemm_fp8(FAKE, 8, 128, FAKE, FAKE, 24, FAKE, FAKE, 1 << 20, None, None) == wq.WQ_ERR_ALIGN
    assert L.wq_gemm_fp8(FAKE, 8, 128, FAKE, FAKE, 16, FAKE, FAKE, 0, None, None) == wq.WQ_ERR_WORKSPACE
    assert L.wq_gemm_fp8(FAKE, 8, 128, None, FAKE, 16, FAKE, FAKE, 1 << 20, None, None) == wq.WQ_ERR_ARG


def test_gptq_validation(L):
    q = L.wq_gptq_quantize
    assert q(FAKE, 1, 8, 256, FAKE, 64, 1, FAKE, FAKE, None, FAKE, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert q(FAKE, 1, 8, 200, FAKE, 128, 1, FAKE, FAKE, None, FAKE, 1 << 20, None) == wq.WQ_ERR_ALIGN
    assert q(FAKE, 1, 8, 256, FAKE, 128, 0, FAKE, FAKE, None, FAKE, 1 << 20, None) == wq.WQ_ERR_ARG
    assert q(FAKE, 1, 8, 256, FAKE, 128, 1, FAKE, FAKE, None, FAKE, 16, None) == wq.WQ_ERR_WORKSPACE
    assert q(FAKE, 1, 8, 256, None, 128, 1, FAKE, FAKE, None, FAKE, 1 << 20, None) == wq.WQ_ERR_ARG
    assert L.wq_gptq_workspace_bytes(8, 256) == 8 * 256 * 8


def test_w8a16_validation(L):
    assert L.wq_gemm_w8a16(FAKE, 2, 96, FAKE, 0, FAKE, 16, FAKE, None) == wq.WQ_ERR_ALIGN   # K % 64
    assert L.wq_gemm_w8a16(FAKE, 2, 128, FAKE, 2, FAKE, 16, FAKE, None) == wq.WQ_ERR_ARG    # format
    assert L.wq_gemm_w8a16(FAKE, 2, 128, None, 1, FAKE, 16, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_gemm_w8a16(FAKE, -1, 128, FAKE, 1, FAKE, 16, FAKE, None) == wq.WQ_ERR_ARG
    assert L.wq_gemm_w8a16(MISALIGNED, 2, 128, FAKE, 0, FAKE, 16, FAKE, None) == wq.WQ_ERR_ALIGN
    assert L.wq_gemm_w8a16(FAKE, 0, 128, FAKE, 0, FAKE, 16, FAKE, None) == wq.WQ_OK


def test_binding_rejects_non_bf16_activations():
    """Entry points whose X and Y are bf16 by contract (no dtype argument)
    refuse other dtypes in the binding, before any pointer is passed."""
    X16 = torch.zeros((2, 16), dtype=torch.float16)
    q = torch.zeros((2, 16), dtype=torch.int8)
    s = torch.zeros((2,), dtype=torch.float32)
    with pytest.raises(wq.WQError) as e:
        wq.wq_quant_act_i8(X16, q, s)
    assert e.value.status == wq.WQ_ERR_ARG and "bfloat16" in str(e.value)
    with pytest.raises(wq.WQError):
        wq.wq_gemm_w4a16(X16, q, s, None, 8, 128, True, X16)


def test_binding_refuses_short_buffers():
    """Every buffer's extent is checked against the sizes the call passes,
    before any pointer reaches the library (the C ABI cannot see extents)."""
    X = torch.zeros((4, 256), dtype=torch.bfloat16)
    codes = torch.zeros((8, 64), dtype=torch.uint8)        # needs [8, 128]
    scales = torch.zeros((8, 2), dtype=torch.float16)
    Y = torch.zeros((4, 8), dtype=torch.bfloat16)
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w4a16(X, codes, scales, None, 8, 128, True, Y)
    assert e.value.status == wq.WQ_ERR_ARG and "codes" in str(e.value)
    W = torch.zeros((8, 256), dtype=torch.bfloat16)
    with pytest.raises(wq.WQError) as e:
        wq.wq_quantize_pack(W, 128, 4, True, torch.zeros((8, 128), dtype=torch.uint8),
                            torch.zeros((8, 1), dtype=torch.float16))
    assert "scales" in str(e.value)
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w8a16(X, torch.zeros((8, 256), dtype=torch.int8), 0,
                         torch.zeros(8, dtype=torch.float32), torch.zeros((4, 4), dtype=torch.bfloat16))
    assert "Y" in str(e.value)
    with pytest.raises(wq.WQError) as e:
        wq.wq_quant_act_i8(X, torch.zeros((4, 256), dtype=torch.int8), torch.zeros(3))
    assert "s holds" in str(e.value)


def test_helpers_allocate_what_the_calls_touch():
    """The allocating helpers pass the extent checks: with CPU tensors every
    call stops only at the device check (no CPU fallback)."""
    N, K, M = 16, 256, 4
    bf = torch.bfloat16
    W, X = torch.zeros(N, K, dtype=bf), torch.zeros(M, K, dtype=bf)
    codes = torch.zeros(N, K // 2, dtype=torch.uint8)
    sc = torch.zeros(N, K // 128, dtype=torch.float16)
    q8, s8 = torch.zeros(N, K, dtype=torch.int8), torch.zeros(N)
    U = torch.zeros(K, K, dtype=torch.float64)
    calls = [
        lambda: wq.quantize_pack(W, 128, 4, True), lambda: wq.quantize_pack(W, 128, 4, False),
        lambda: wq.quantize_pack(W, K, 8, True),
        lambda: wq.dequant(codes, sc, sc, K, 128, 4, False, torch.float32),
        lambda: wq.dequant(q8, s8, None, K, K, 8, True, bf),
        lambda: wq.gemm_w4a16(X, codes, sc, sc, 128, False),
        lambda: wq.quant_act_i8(X), lambda: wq.gemm_w8a8(X, q8, s8, want_acc=True),
        lambda: wq.channel_absmax(X), lambda: wq.smooth_scales(torch.zeros(K), torch.zeros(K)),
        lambda: wq.quantize_i8_smooth(W, torch.zeros(K)),
        lambda: wq.quant_act_i8_smooth(X, torch.zeros(K)),
        lambda: wq.gemm_w8a8_smooth(X, q8, s8, torch.zeros(K)),
        lambda: wq.quant_kv(torch.zeros(2, 8, 128, dtype=bf), torch.zeros(2, 8, 128, dtype=bf)),
        lambda: wq.quantize_fp8_rows(W),
        lambda: wq.gemm_fp8(X, torch.zeros(N, K, dtype=torch.uint8), s8),
        lambda: wq.gemm_w8a16(X, q8, s8),
        lambda: wq.gptq_quantize(W, U, True), lambda: wq.gptq_quantize(W, U, False),
    ]
    for call in calls:
        with pytest.raises(wq.WQError) as e:
            call()
        assert "CUDA device" in str(e.value)
