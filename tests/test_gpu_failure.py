"""Failure detection on the GPU without a GPU fault: the bounded wait every kernel uses on
its asynchronous copies gives up after its limit, records LLSA_ERR_TIMEOUT in the device
status word and lets the kernel return; the context stays usable and the next call is clean.

The wait is made to run out on an mbarrier armed for bytes that no copy delivers (no copy
is issued at all), through llsa_check_bounded_wait."""
import pytest
import torch

from log_linear_hierarchical_b200 import api
from llsa_testlib import check_pyramid_bitexact, inputs_for, run_gpu

pytestmark = pytest.mark.gpu

LLSA_ERR_TIMEOUT = 6


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("limit", [2_000, 200_000])
def test_wait_that_runs_out_records_timeout_and_returns(limit):
    assert api.llsa_device_status() == 0
    api.llsa_check_bounded_wait(limit)
    torch.cuda.synchronize()                      # the kernel returned
    assert api.llsa_device_status() == LLSA_ERR_TIMEOUT
    assert api.llsa_device_status() == 0          # read and cleared


def test_next_call_after_a_timeout_is_clean():
    api.llsa_check_bounded_wait(5_000)
    assert api.llsa_device_status() == LLSA_ERR_TIMEOUT
    inputs = inputs_for(1, 2, 4096, 64, "bf16", "smooth", 31)
    gpu = run_gpu(1, 2, 4096, 64, 4, 2, "bf16", inputs)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, 2)
