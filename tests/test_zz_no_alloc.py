"""The allocation-free weight-gradient entry point, on the GPU.

dwconv2d_bwd_weight_noalloc is for callers that cannot allocate device
memory where they call it: programs whose device memory is an arena reserved
up front, and latency-critical paths where cudaMalloc / cudaFree are not
acceptable because they can synchronise the device.  Its scratch is a fixed
array inside the library.  This test calls it through the C ABI and checks it
against dwconv2d_bwd_weight with a caller workspace, on two calls in a row
(the second call starts from the scratch the first one left behind), within
the tolerance of the other parity tests: 1e-5 of the sum of the magnitudes of
the terms of each gradient element.  The file is collected last so that a run
stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200 import build as dwbuild
from depthwise_convolution_fwd_b200.workloads import Case
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

CASES = [
    Case("na_nhwc_3x3", 4, 40, 44, 64, 3, 3, seed=91),                   # tiled kernels
    Case("na_nhwc_1x31", 8, 2, 200, 64, 1, 31, act="normal", seed=92),   # tiled, 8 MiB scratch
    Case("na_nchw_5x5_s2", 2, 21, 19, 12, 5, 5, stride=2, layout="nchw", seed=93),  # direct
]


@pytest.fixture(scope="module")
def library():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    dwbuild.build()
    return dw.lib()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_noalloc_matches_workspace_entry_point_twice(library, case):
    inp = gu.inputs(case)
    x, dy = inp["x"].cuda(), inp["dy"].cuda()
    kw = dict(stride=case.stride, dilation=case.dilation, padding=case.padding,
              layout=case.layout)
    ref_w, ref_b = dw.dwconv2d_bwd_weight(x, dy, (case.kH, case.kW), **kw)
    torch.cuda.synchronize()
    p = gu.problem(case)
    scale_w, scale_b = oracle.bwd_weight(p, np.abs(gu.f64(inp["x"])), np.abs(gu.f64(inp["dy"])))
    desc = gu.desc_of(case)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        got_w = torch.full((case.C, case.kH, case.kW), float("nan"), device="cuda")
        got_b = torch.full((case.C,), float("nan"), device="cuda")
        st = library.dwconv2d_bwd_weight_noalloc(ctypes.byref(desc), x.data_ptr(), dy.data_ptr(),
                                                 got_w.data_ptr(), got_b.data_ptr(), stream)
        assert st == dw.DW_OK, dw.status_string(st)
        torch.cuda.synchronize()
        gu.assert_close(got_w.cpu().numpy(), ref_w.cpu().numpy(), scale_w,
                        f"{case.name} dW, call {call + 1}")
        gu.assert_close(got_b.cpu().numpy(), ref_b.cpu().numpy(), scale_b,
                        f"{case.name} db, call {call + 1}")
    assert dw.dwconv2d_take_device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch(library):
    """A problem whose scratch exceeds the fixed array is refused with
    DW_ERR_TOO_LARGE before any buffer is touched (the pointers below are
    small real buffers, never read)."""
    desc = dw.make_desc(1, 256, 256, 1 << 14, 3, 3, layout="nchw")
    assert dw.dwconv2d_bwd_weight_workspace_size(desc) > dw.DW_NOALLOC_SCRATCH_BYTES
    buf = torch.empty(1024, device="cuda")
    st = library.dwconv2d_bwd_weight_noalloc(ctypes.byref(desc), buf.data_ptr(),
                                             buf.data_ptr() + 1024, buf.data_ptr() + 2048, None,
                                             torch.cuda.current_stream().cuda_stream)
    assert st == dw.DW_ERR_TOO_LARGE
