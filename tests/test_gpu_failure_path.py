"""The failure path on a GPU, without faulting it: a kernel whose bounded
wait on an asynchronous-copy barrier never completes gives up after its
limit (or when another warp raises the CTA's abort flag), records
DW_ERR_DEVICE_TIMEOUT in the library's device error word and returns; the
context stays usable and the next calls are correct."""
import time

import pytest
import torch

import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200 import build as dwbuild
from depthwise_convolution_fwd_b200.workloads import Case
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dwbuild.build()
    dw.lib()
    torch.cuda.synchronize()
    assert dw.dwconv2d_take_device_error() == 0
    yield


@pytest.mark.parametrize("mode", [0, 1])
def test_bounded_wait_reports_timeout(mode):
    s = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    assert dw.selftest_wait_timeout_raw(mode, 2000, s) == dw.DW_OK
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert dw.dwconv2d_take_device_error() == dw.DW_ERR_DEVICE_TIMEOUT
    assert dw.dwconv2d_take_device_error() == 0          # reading clears the word
    assert elapsed < 1.5                                 # it gave up, it did not hang
    # the context is still good: a normal call after the timeout is correct
    case = Case("after_timeout", 2, 20, 24, 32, 3, 3, seed=77)
    inp = gu.inputs(case)
    ref, scale = gu.reference_fwd(case, inp)
    y = gu.gpu_fwd(case, inp)
    torch.cuda.synchronize()
    gu.assert_close(y.cpu().numpy(), ref, scale, "forward after a timed-out wait")
    assert dw.dwconv2d_take_device_error() == 0
