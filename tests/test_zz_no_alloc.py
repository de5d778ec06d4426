"""The decode product without allocation (wq_gemm_w4a16_noalloc), checked
against the fp64 oracle and against the workspace entry point.

Some callers cannot hand the library a device workspace: a serving loop
whose device memory is owned by another allocator under a fixed budget, a
plain C host with no device allocator, or a latency-critical path where a
cudaMalloc (which may synchronize the device) is not acceptable.  For them
wq_gemm_w4a16_noalloc keeps its scratch in an array inside the library's own
device image.  Every call shares that array, which keeps the last call's
contents, so the entry point clears the arrival counters itself.  This file is
collected last: it must pass alone in a fresh process as well as after every
other test.
"""
import ctypes

import pytest
import torch

import bit_gemm_group_b200 as wq
import oracle
from parity_util import REL_ROW_TOL, oracle_input, rel_row_error
from workloads import bf16_bits, make_activation, make_weight

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(L, X, codes, scales, zeros, N, sym, Y):
    M, K = X.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.wq_gemm_w4a16_noalloc(_p(X), M, K, _p(codes), _p(scales), _p(zeros), N, 128,
                                   int(sym), _p(Y), stream)


def _case(N, K, M, sym):
    W = make_weight(N, K, 0.02, seed=N + K, outlier_frac=0.001, outlier_scale=30.0)
    codes, scales, zeros = wq.quantize_pack(W.cuda(), 128, 4, sym)
    arr, tag = oracle_input(W)
    oc, osc, oz, st = oracle.quantize_int4(arr, 128, sym, dtype_tag=tag)
    assert st == oracle.OK
    X = make_activation(M, K, seed=M)
    return X, (codes, scales, zeros), (oc, osc, oz)


def _windows(N):
    return [(0, N)] if N <= 1024 else [(0, 256), (N // 2 - 128, N // 2 + 128), (N - 256, N)]


# M = 1, 2 run the CUDA-core kernel (no scratch); M >= 3 the tensor-core
# kernel, whose arrival counters and (for K > 2048) K-range partials live in
# the scratch array
@pytest.mark.parametrize("N,K,M,sym", [(4096, 4096, 1, True), (11008, 4096, 2, False),
                                       (8000, 11008, 16, True), (136, 1152, 3, False),
                                       (136, 1152, 9, True), (264, 4096, 16, False),
                                       (28672, 8192, 4, False)])
def test_noalloc_matches_oracle_on_two_calls(N, K, M, sym):
    L = wq.lib()
    X, dq, oq = _case(N, K, M, sym)
    codes, scales, zeros = dq
    Xd = X.cuda()
    wq.wq_get_device_status(reset=True)
    outs = []
    for _ in range(2):  # two calls in a row share (and must clear) the scratch
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(L, Xd, codes, scales, zeros, N, sym, Y) == wq.WQ_OK
        torch.cuda.synchronize()
        outs.append(Y.float().cpu().numpy())
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK
    for n0, n1 in _windows(N):
        ref, st = oracle.gemm_w4a16(bf16_bits(X), *oq, 128, sym, n0, n1)
        assert st == oracle.OK
        for Yh in outs:
            err = rel_row_error(Yh[:, n0:n1], ref, rounding_aware=N < 256)
            assert err <= REL_ROW_TOL, (n0, n1, err)
    # the workspace entry point computes the same product
    Y_ws = wq.gemm_w4a16(Xd, codes, scales, zeros, 128, sym).float().cpu().numpy()
    assert (outs[0] == Y_ws).all() and (outs[1] == Y_ws).all()


def test_noalloc_result_unchanged_by_a_call_on_another_shape():
    """The scratch keeps the last call's contents: a call on another shape in
    between must not change the next result."""
    L = wq.lib()
    Xa, (ca, sa, za), _ = _case(8000, 11008, 8, False)
    Xb, (cb, sb, zb), _ = _case(264, 4096, 13, True)
    Xa, Xb = Xa.cuda(), Xb.cuda()
    Ya1 = torch.empty((8, 8000), dtype=torch.bfloat16, device="cuda")
    Ya2 = torch.empty_like(Ya1)
    Yb = torch.empty((13, 264), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(L, Xa, ca, sa, za, 8000, False, Ya1) == wq.WQ_OK
    assert _call_noalloc(L, Xb, cb, sb, zb, 264, True, Yb) == wq.WQ_OK
    assert _call_noalloc(L, Xa, ca, sa, za, 8000, False, Ya2) == wq.WQ_OK
    torch.cuda.synchronize()
    assert torch.equal(Ya1, Ya2)
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
