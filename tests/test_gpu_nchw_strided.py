"""GPU parity of the NCHW stride-2 forward (2-D tiles with the stride in the
index map) against the float64 oracle: every column phase of the box start,
SAME and explicit pads, ragged output edges, the fused epilogue and 16-bit
activations; the input gradient of the same shapes (direct kernel) too."""
import numpy as np
import pytest
import torch

import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200 import build as dwbuild
from depthwise_convolution_fwd_b200.workloads import Case
from tests import gpu_util as gu
from tests import test_gpu_fused_epilogue as fe
from tests import test_gpu_half_activations as ha

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dwbuild.build()
    dw.lib()
    yield
    torch.cuda.synchronize()
    assert dw.dwconv2d_take_device_error() == 0


CASES = [
    Case("s2_pad1", 2, 29, 40, 12, 3, 3, stride=2, padding=1, layout="nchw", seed=501),
    Case("s2_same", 2, 30, 40, 6, 3, 3, stride=2, layout="nchw", seed=502),
    Case("s2_pl3", 1, 33, 48, 5, 3, 3, stride=2, padding=(2, 1, 3, 0), layout="nchw", seed=503),
    Case("s2_pl2", 1, 21, 44, 7, 3, 3, stride=2, padding=(0, 0, 2, 2), layout="nchw", seed=504),
    Case("s2_wide", 1, 9, 300, 3, 3, 3, stride=2, padding=1, layout="nchw", seed=505),
    Case("s2_mobilenet_c8", 4, 56, 56, 8, 3, 3, stride=2, padding=1, layout="nchw", seed=506),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_nchw_stride2_forward(case):
    inp = gu.inputs(case)
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    assert gu.chosen_algo(case, 0, inp["x"].cuda(), inp["w"].cuda(), y) == dw.DW_ALGO_TILED
    ref, scale = gu.reference_fwd(case, inp)
    for algo in ("tiled", "direct"):
        got = gu.gpu_fwd(case, inp, algo)
        torch.cuda.synchronize()
        gu.assert_close(got.cpu().numpy(), ref, scale, f"{case.name} fwd [{algo}]")
    dxr, dxs = gu.reference_bwd(case, inp)
    dx = gu.gpu_bwd(case, inp)
    torch.cuda.synchronize()
    gu.assert_close(dx.cpu().numpy(), dxr, dxs, f"{case.name} bwd")


# input gradient tiles: both pad parities in each direction, ragged dx widths
BWD = [
    Case("b2_pad1", 2, 29, 40, 12, 3, 3, stride=2, padding=1, layout="nchw", seed=511),
    Case("b2_p00", 1, 30, 40, 5, 3, 3, stride=2, padding=(0, 1, 0, 1), layout="nchw", seed=512),
    Case("b2_p10", 1, 27, 40, 5, 3, 3, stride=2, padding=(1, 0, 0, 1), layout="nchw", seed=513),
    Case("b2_p01", 2, 22, 40, 3, 3, 3, stride=2, padding=(0, 1, 1, 0), layout="nchw", seed=514),
    Case("b2_pl3", 1, 25, 36, 7, 3, 3, stride=2, padding=(2, 1, 3, 2), layout="nchw", seed=515),
    Case("b2_w39", 1, 17, 39, 4, 3, 3, stride=2, padding=1, layout="nchw", seed=516),
    Case("b2_wide", 1, 12, 296, 3, 3, 3, stride=2, padding=(1, 1, 1, 0), layout="nchw", seed=517),
]


@pytest.mark.parametrize("case", BWD, ids=lambda c: c.name)
def test_nchw_stride2_input_gradient_tiles(case):
    inp = gu.inputs(case)
    dy, w = inp["dy"].cuda(), inp["w"].cuda()
    dx = torch.empty(case.in_shape(), device="cuda")
    assert gu.chosen_algo(case, 1, dy, w, dx) == dw.DW_ALGO_TILED
    ref, scale = gu.reference_bwd(case, inp)
    for algo in ("tiled", "direct"):
        got = gu.gpu_bwd(case, inp, algo)
        torch.cuda.synchronize()
        gu.assert_close(got.cpu().numpy(), ref, scale, f"{case.name} bwd [{algo}]")


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: c.name)
def test_nchw_stride2_fused(case):
    inp = gu.inputs(case)
    bn = fe.bn_of(case)
    for act in ("relu6", "silu"):
        ref, tol = fe.bound(case, inp, bn, act)
        fe.check_close(fe.gpu_fused(case, inp, bn, act), ref, tol, f"{case.name} fused {act}")


@pytest.mark.parametrize("name", ["f16", "bf16"])
def test_nchw_stride2_half(name):
    case = Case("s2_half", 2, 29, 48, 6, 3, 3, stride=2, padding=1, layout="nchw", seed=507)
    ha.run_case(case, name, "auto")


def test_nchw_stride2_full_size_sampled():
    case = Case("mobilenet_nchw_s2", 32, 56, 56, 144, 3, 3, stride=2, padding=1, layout="nchw",
                seed=1102)
    rng = np.random.default_rng(41)
    inp = gu.inputs(case)
    y = gu.gpu_fwd(case, inp)
    torch.cuda.synchronize()
    idx = gu.structured_sample(tuple(y.shape), case.layout, rng, count=4000)
    ref, scale = gu.reference_fwd_at(case, inp, idx)
    gu.assert_close(y.reshape(-1)[torch.from_numpy(idx).cuda()].cpu().numpy(), ref, scale,
                    "mobilenet nchw stride 2 sampled")
    dx = gu.gpu_bwd(case, inp)
    torch.cuda.synchronize()
    idx = gu.structured_sample(tuple(dx.shape), case.layout, rng, count=4000)
    ref, scale = gu.reference_bwd_at(case, inp, idx)
    gu.assert_close(dx.reshape(-1)[torch.from_numpy(idx).cuda()].cpu().numpy(), ref, scale,
                    "mobilenet nchw stride 2 input gradient sampled")
