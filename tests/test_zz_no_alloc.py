"""The decode product without allocation (wq_gemm_w4a16_noalloc) against the
workspace entry point (wq_gemm_w4a16).

Callers that cannot allocate device memory -- code running during CUDA graph
capture, serving loops whose memory belongs to another allocator, plain C
hosts -- use wq_gemm_w4a16_noalloc, which keeps its scratch in an array inside
the library's device image.  This file is collected last; it must pass alone in
a fresh process as well as after every other test (the array keeps the last
call's contents, so the entry point has to clear what must start at zero).
"""
import ctypes

import pytest
import torch

import bit_gemm_group_b200 as wq
from parity_util import REL_ROW_TOL, rel_row_error
from workloads import make_activation, make_weight

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(L, X, codes, scales, zeros, N, sym, Y):
    M, K = X.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.wq_gemm_w4a16_noalloc(_p(X), M, K, _p(codes), _p(scales), _p(zeros), N, 128,
                                   int(sym), _p(Y), stream)


@pytest.mark.parametrize("N,K,M,sym", [(4096, 4096, 1, True), (11008, 4096, 4, False),
                                       (8000, 11008, 16, True), (136, 1152, 3, False)])
def test_noalloc_matches_workspace_entry_point(N, K, M, sym):
    L = wq.lib()
    W = make_weight(N, K, 0.02, seed=N + K, outlier_frac=0.001, outlier_scale=30.0).cuda()
    codes, scales, zeros = wq.quantize_pack(W, 128, 4, sym)
    X = make_activation(M, K, seed=M).cuda()
    wq.wq_get_device_status(reset=True)
    Y_ref = wq.gemm_w4a16(X, codes, scales, zeros, 128, sym).float().cpu().numpy()
    for _ in range(2):  # two calls in a row share (and must clear) the scratch
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(L, X, codes, scales, zeros, N, sym, Y) == wq.WQ_OK
        torch.cuda.synchronize()
        err = rel_row_error(Y.float().cpu().numpy(), Y_ref, rounding_aware=N < 256)
        assert err <= REL_ROW_TOL, err
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK


def test_noalloc_rejects_beyond_its_limits():
    L = wq.lib()
    X = torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((64, 128), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((64, 2), dtype=torch.float16, device="cuda")
    Y = torch.zeros((17, 64), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(L, X, codes, scales, None, 64, True, Y) == wq.WQ_ERR_UNSUPPORTED
    big_n = 131072 + 8
    assert L.wq_gemm_w4a16_noalloc(_p(X[:1]), 1, 256, _p(codes), _p(scales), None, big_n, 128, 1,
                                   _p(Y), None) == wq.WQ_ERR_UNSUPPORTED
