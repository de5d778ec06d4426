"""Failure detection without a GPU fault: a bounded wait that nothing will
satisfy gives up after its limit, records WQ_ERR_TIMEOUT in the device status
word and returns; the context stays usable afterwards."""
import pytest
import torch

import bit_gemm_group_b200 as wq
from workloads import make_weight

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    wq.wq_get_device_status(reset=True)
    wq.wq_selftest_wait_timeout(2000)
    assert wq.wq_get_device_status(reset=True) == wq.WQ_ERR_TIMEOUT
    W = make_weight(16, 256, 0.02, seed=0).cuda()
    codes, scales, _ = wq.quantize_pack(W, 128, 4, True)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status(reset=True) == wq.WQ_OK
    assert codes.shape == (16, 128)


def test_selftest_rejects_bad_limit():
    with pytest.raises(wq.WQError):
        wq.wq_selftest_wait_timeout(0)
