"""GPU parity of the channel multiplier (C input channels, C*M outputs,
output o reads input o // M) against the float64 oracle: forward, input
gradient, weight and bias gradients and the fused epilogue, on the tiled NHWC
kernels (M = 2 and 4, 3x3 and 5x5 filters), the tiled NCHW kernels (one input
plane feeding its M output planes, M dy planes summed into one dx plane, or
one output plane per tile) and the direct kernels.
Error rule as for the plain calls: |gpu - ref| <= 1e-5 * sum|terms|, exact
where there is no term."""
import numpy as np
import pytest
import torch

import oracle
import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200 import build as dwbuild
from depthwise_convolution_fwd_b200 import workloads as wl
from depthwise_convolution_fwd_b200.workloads import Case
from tests import gpu_util as gu
from tests import test_gpu_fused_epilogue as fe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dwbuild.build()
    dw.lib()
    yield
    torch.cuda.synchronize()
    assert dw.dwconv2d_take_device_error() == 0


def check_all(case, fwd_algos=("auto", "direct")):
    inp = gu.inputs(case)
    ref, scale = gu.reference_fwd(case, inp)
    for algo in fwd_algos:
        y = gu.gpu_fwd(case, inp, algo)
        torch.cuda.synchronize()
        gu.assert_close(y.cpu().numpy(), ref, scale, f"{case.name} fwd [{algo}]")
    dxr, dxs = gu.reference_bwd(case, inp)
    dx = gu.gpu_bwd(case, inp)
    torch.cuda.synchronize()
    gu.assert_close(dx.cpu().numpy(), dxr, dxs, f"{case.name} bwd_input")
    p = gu.problem(case)
    x, dy = gu.f64(inp["x"]), gu.f64(inp["dy"])
    dwr, dbr = oracle.bwd_weight(p, x, dy)
    dws, dbs = oracle.bwd_weight(p, np.abs(x), np.abs(dy))
    g_w, g_b = dw.dwconv2d_bwd_weight(inp["x"].cuda(), inp["dy"].cuda(), (case.kH, case.kW),
                                      stride=case.stride, dilation=case.dilation,
                                      padding=case.padding, layout=case.layout)
    torch.cuda.synchronize()
    gu.assert_close(g_w.cpu().numpy(), dwr, dws, f"{case.name} dW")
    gu.assert_close(g_b.cpu().numpy(), dbr, dbs, f"{case.name} db")
    bn = fe.bn_of(case)
    for act in ("relu6", "silu"):
        r, tol = fe.bound(case, inp, bn, act)
        fe.check_close(fe.gpu_fused(case, inp, bn, act), r, tol, f"{case.name} fused {act}")


TILED = [
    Case("m2_3x3", 2, 19, 37, 20, 3, 3, multiplier=2, seed=301),
    Case("m4_3x3", 2, 17, 40, 12, 3, 3, multiplier=4, seed=302),
    Case("m2_3x3_s2", 3, 29, 31, 36, 3, 3, stride=2, padding=1, multiplier=2, seed=303),
    Case("m4_3x3_s2_same", 2, 30, 33, 8, 3, 3, stride=2, multiplier=4, seed=304),
    Case("m2_5x5", 2, 23, 21, 28, 5, 5, multiplier=2, seed=305),
    Case("m4_5x5_pad", 1, 26, 35, 16, 5, 5, padding=(1, 3, 0, 2), multiplier=4, seed=306),
    Case("m2_many_tiles", 8, 64, 64, 64, 3, 3, multiplier=2, seed=307),
]


@pytest.mark.parametrize("case", TILED, ids=lambda c: c.name)
def test_tiled_multiplier_forward(case):
    inp = gu.inputs(case)
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    assert gu.chosen_algo(case, 0, inp["x"].cuda(), inp["w"].cuda(), y) == dw.DW_ALGO_TILED
    assert gu.chosen_algo(case, 2, inp["x"].cuda(), y, inp["w"].cuda()) == dw.DW_ALGO_TILED
    check_all(case, fwd_algos=("tiled", "direct"))
    # the direct weight gradient agrees too
    p = gu.problem(case)
    x, dy = gu.f64(inp["x"]), gu.f64(inp["dy"])
    dwr, dbr = oracle.bwd_weight(p, x, dy)
    dws, dbs = oracle.bwd_weight(p, np.abs(x), np.abs(dy))
    g_w, g_b = dw.dwconv2d_bwd_weight(inp["x"].cuda(), inp["dy"].cuda(), (case.kH, case.kW),
                                      stride=case.stride, dilation=case.dilation,
                                      padding=case.padding, layout=case.layout, algo="direct")
    torch.cuda.synchronize()
    gu.assert_close(g_w.cpu().numpy(), dwr, dws, f"{case.name} dW direct")
    gu.assert_close(g_b.cpu().numpy(), dbr, dbs, f"{case.name} db direct")


DIRECT = [
    Case("m3_3x3", 2, 11, 13, 5, 3, 3, multiplier=3, seed=311),
    Case("m2_nchw", 2, 12, 16, 6, 3, 3, multiplier=2, layout="nchw", seed=312),
    Case("m3_nchw_s2_d2", 1, 15, 17, 4, 3, 3, stride=2, dilation=2, multiplier=3,
         layout="nchw", seed=313),
    Case("m2_odd_c", 2, 9, 10, 7, 5, 5, multiplier=2, seed=314),
    Case("m5_1x7", 2, 3, 40, 4, 1, 7, multiplier=5, act="normal", seed=315),
    Case("m8_7x7", 1, 14, 12, 4, 7, 7, multiplier=8, seed=316),
]


@pytest.mark.parametrize("case", DIRECT + wl.multiplier()[:1], ids=lambda c: c.name)
def test_direct_multiplier(case):
    check_all(case)


def test_f16_weights_bit_identical():
    case = TILED[0].with_(wtype="f16")
    inp = gu.inputs(case)
    a = gu.gpu_fwd(case, inp, w_key="w")
    b = gu.gpu_fwd(case, inp, w_key="w32")
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_multiplier_one_matches_plain_call():
    case = Case("m1", 2, 20, 24, 32, 3, 3, seed=320)
    inp = gu.inputs(case)
    desc1 = gu.desc_of(case)
    desc1.multiplier = 1
    x, w, b = inp["x"].cuda(), inp["w"].cuda(), inp["b"].cuda()
    y0 = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    y1 = torch.empty_like(y0)
    d0 = gu.desc_of(case)
    d0.multiplier = 0
    s = torch.cuda.current_stream().cuda_stream
    assert dw.fwd_raw(d0, x.data_ptr(), w.data_ptr(), b.data_ptr(), y0.data_ptr(), s) == 0
    assert dw.fwd_raw(desc1, x.data_ptr(), w.data_ptr(), b.data_ptr(), y1.data_ptr(), s) == 0
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("case", [c for c in wl.multiplier() if c.H == 512], ids=lambda c: c.name)
def test_full_size_sampled(case):
    rng = np.random.default_rng(23)
    inp = gu.inputs(case)
    y = gu.gpu_fwd(case, inp)
    dx = gu.gpu_bwd(case, inp)
    torch.cuda.synchronize()
    idx = gu.structured_sample(tuple(y.shape), case.layout, rng, count=4000)
    ref, scale = gu.reference_fwd_at(case, inp, idx)
    gu.assert_close(y.reshape(-1)[torch.from_numpy(idx).cuda()].cpu().numpy(), ref, scale,
                    f"{case.name} fwd sampled")
    idx = gu.structured_sample(tuple(dx.shape), case.layout, rng, count=4000)
    ref, scale = gu.reference_bwd_at(case, inp, idx)
    gu.assert_close(dx.reshape(-1)[torch.from_numpy(idx).cuda()].cpu().numpy(), ref, scale,
                    f"{case.name} bwd sampled")


@pytest.mark.parametrize("case", [c for c in TILED if c.kH == 3], ids=lambda c: c.name)
def test_tiled_multiplier_input_gradient(case):
    inp = gu.inputs(case)
    dy, w = inp["dy"].cuda(), inp["w"].cuda()
    dx = torch.empty(case.in_shape(), device="cuda")
    assert gu.chosen_algo(case, 1, dy, w, dx) == dw.DW_ALGO_TILED
    ref, scale = gu.reference_bwd(case, inp)
    for algo in ("tiled", "direct"):
        got = gu.gpu_bwd(case, inp, algo)
        torch.cuda.synchronize()
        gu.assert_close(got.cpu().numpy(), ref, scale, f"{case.name} bwd_input [{algo}]")


NCHW_TILED = [
    Case("mn2_3x3", 2, 21, 40, 6, 3, 3, multiplier=2, layout="nchw", seed=331),
    Case("mn4_5x5", 1, 19, 96, 3, 5, 5, multiplier=4, layout="nchw", seed=332),
    Case("mn3_7x7", 1, 17, 36, 2, 7, 7, multiplier=3, layout="nchw", seed=333),
    Case("mn2_s2", 2, 29, 80, 4, 3, 3, stride=2, padding=1, multiplier=2, layout="nchw", seed=334),
]


@pytest.mark.parametrize("case", NCHW_TILED + [
    Case("mnf4_3x3", 2, 21, 36, 5, 3, 3, padding=(0, 2, 3, 3), multiplier=4, layout="nchw",
         seed=335),
    Case("mnf2_5x5", 2, 35, 44, 3, 5, 5, multiplier=2, layout="nchw", seed=336),
    Case("mnf2_3x3_many", 4, 64, 64, 8, 3, 3, multiplier=2, layout="nchw", seed=337),
    Case("mnf2_s2_same", 2, 30, 72, 3, 3, 3, stride=2, multiplier=2, layout="nchw", seed=338),
], ids=lambda c: c.name)
def test_nchw_multiplier_tiles(case):
    inp = gu.inputs(case)
    x, w = inp["x"].cuda(), inp["w"].cuda()
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    assert gu.chosen_algo(case, 0, x, w, y) == dw.DW_ALGO_TILED
    assert gu.chosen_algo(case, 2, x, y, w) == dw.DW_ALGO_TILED
    check_all(case, fwd_algos=("tiled", "direct"))


# NCHW input gradient with a multiplier: one box of M dy planes per dx tile
# (stride 1; 3x3 with M = 2, 4, 5x5 and 7x7 with M = 2; dy rows a multiple of
# 16 bytes)
NCHW_BWD = [
    Case("mnb2_3x3", 2, 21, 40, 6, 3, 3, multiplier=2, layout="nchw", seed=341),
    Case("mnb4_3x3_pad", 1, 19, 36, 5, 3, 3, padding=(0, 2, 3, 3), multiplier=4,
         layout="nchw", seed=342),
    Case("mnb2_5x5", 2, 35, 48, 3, 5, 5, multiplier=2, layout="nchw", seed=343),
    Case("mnb2_7x7_wide", 1, 17, 260, 2, 7, 7, multiplier=2, layout="nchw", seed=344),
    Case("mnb2_3x3_many", 4, 64, 64, 8, 3, 3, multiplier=2, layout="nchw", seed=345),
]


@pytest.mark.parametrize("case", NCHW_BWD, ids=lambda c: c.name)
def test_nchw_multiplier_input_gradient_tiles(case):
    inp = gu.inputs(case)
    dy, w = inp["dy"].cuda(), inp["w"].cuda()
    dx = torch.empty(case.in_shape(), device="cuda")
    assert gu.chosen_algo(case, 1, dy, w, dx) == dw.DW_ALGO_TILED
    ref, scale = gu.reference_bwd(case, inp)
    for algo in ("tiled", "direct"):
        got = gu.gpu_bwd(case, inp, algo)
        torch.cuda.synchronize()
        gu.assert_close(got.cpu().numpy(), ref, scale, f"{case.name} bwd_input [{algo}]")


@pytest.mark.parametrize("name", ["f16", "bf16"])
@pytest.mark.parametrize("case", [NCHW_BWD[0], NCHW_TILED[1], NCHW_TILED[3]], ids=lambda c: c.name)
def test_nchw_multiplier_half(case, name):
    from tests import test_gpu_half_activations as ha
    dt, _ = ha.DTYPES[name]
    inp = ha.inputs16(case, dt)
    x = inp["x"].cuda()
    Ho, Wo = gu.out_hw(case)
    y = torch.empty(case.out_shape(Ho, Wo), device="cuda", dtype=dt)
    desc = gu.desc_of(case)
    desc.atype = {"f16": dw.DW_F16, "bf16": dw.DW_BF16}[name]
    wp = inp["w"].cuda().data_ptr()
    assert dw.dwconv2d_query_algo(desc, 0, x.data_ptr(), wp, y.data_ptr()) == dw.DW_ALGO_TILED
    if case in NCHW_BWD or case.stride == 2:
        assert dw.dwconv2d_query_algo(desc, 1, y.data_ptr(), wp, x.data_ptr()) == dw.DW_ALGO_TILED
    ha.run_case(case, name, "auto")


# NHWC multiplier tiles with 16-bit activations (C a multiple of 8: rows of
# 16 bytes): forward, input gradient, weight gradient
HALF_TILED = [
    Case("hm2_3x3", 2, 19, 37, 24, 3, 3, multiplier=2, seed=351),
    Case("hm4_3x3", 2, 17, 40, 16, 3, 3, multiplier=4, seed=352),
    Case("hm2_3x3_s2", 3, 29, 31, 40, 3, 3, stride=2, padding=1, multiplier=2, seed=353),
    Case("hm4_3x3_s2_same", 2, 30, 33, 8, 3, 3, stride=2, multiplier=4, seed=354),
    Case("hm2_5x5", 2, 23, 21, 32, 5, 5, multiplier=2, seed=355),
]


@pytest.mark.parametrize("name", ["f16", "bf16"])
@pytest.mark.parametrize("case", HALF_TILED, ids=lambda c: c.name)
def test_nhwc_multiplier_half_tiles(case, name):
    from tests import test_gpu_half_activations as ha
    dt, _ = ha.DTYPES[name]
    inp = ha.inputs16(case, dt)
    x, g = inp["x"].cuda(), inp["dy"].cuda()
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda", dtype=dt)
    desc = gu.desc_of(case)
    desc.atype = {"f16": dw.DW_F16, "bf16": dw.DW_BF16}[name]
    wp = inp["w"].cuda().data_ptr()
    assert dw.dwconv2d_query_algo(desc, 0, x.data_ptr(), wp, y.data_ptr()) == dw.DW_ALGO_TILED
    if case.kH == 3:
        assert dw.dwconv2d_query_algo(desc, 1, y.data_ptr(), wp, x.data_ptr()) == dw.DW_ALGO_TILED
    gw = torch.empty(case.multiplier * case.C, case.kH, case.kW, device="cuda")
    assert dw.dwconv2d_query_algo(desc, 2, x.data_ptr(), g.data_ptr(), gw.data_ptr()) == dw.DW_ALGO_TILED
    ha.run_case(case, name, "auto")
