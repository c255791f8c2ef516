"""GPU parity of the weight and bias gradients against the float64 oracle.

Rule as for the other calls: |gpu - ref| <= 1e-5 * sum|terms| per element,
the scale being the oracle's gradient of |x| and |dy| (every term
non-negative), exact where there is no term.  Both kernel families; calls
repeat bit-identically (fixed reduction order)."""
import numpy as np
import pytest
import torch

import oracle
import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200 import build as dwbuild
from depthwise_convolution_fwd_b200 import workloads as wl
from depthwise_convolution_fwd_b200.workloads import Case
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dwbuild.build()
    dw.lib()
    yield
    torch.cuda.synchronize()
    assert dw.dwconv2d_take_device_error() == 0


def reference(case, inp):
    p = gu.problem(case)
    x, dy = gu.f64(inp["x"]), gu.f64(inp["dy"])
    dwr, dbr = oracle.bwd_weight(p, x, dy)
    dws, dbs = oracle.bwd_weight(p, np.abs(x), np.abs(dy))
    return dwr, dbr, dws, dbs


def gpu(case, inp, algo="auto"):
    return dw.dwconv2d_bwd_weight(inp["x"].cuda(), inp["dy"].cuda(), (case.kH, case.kW),
                                  stride=case.stride, dilation=case.dilation,
                                  padding=case.padding, layout=case.layout, algo=algo)


def check(case, algos=("auto", "direct")):
    inp = gu.inputs(case)
    dwr, dbr, dws, dbs = reference(case, inp)
    for algo in algos:
        g_w, g_b = gpu(case, inp, algo)
        torch.cuda.synchronize()
        gu.assert_close(g_w.cpu().numpy(), dwr, dws, f"{case.name} dW [{algo}]")
        gu.assert_close(g_b.cpu().numpy(), dbr, dbs, f"{case.name} db [{algo}]")


CONFIGS = wl.tiny() + wl.mobilenet() + [c for c in wl.conformer() if c.W == 24] + \
    [c for c in wl.large() if c.H == 30] + [c for c in wl.edge() if c.wtype == "f32"]


@pytest.mark.parametrize("case", CONFIGS, ids=lambda c: c.name)
def test_config_cases(case):
    check(case)


TILED = [
    Case("w_3x3_s1", 3, 37, 45, 72, 3, 3, seed=71),
    Case("w_3x3_s1_pad", 2, 23, 70, 36, 3, 3, padding=(0, 2, 2, 1), seed=72),
    Case("w_3x3_s2", 4, 29, 41, 44, 3, 3, stride=2, padding=1, seed=73),
    Case("w_3x3_s2_same", 2, 30, 34, 40, 3, 3, stride=2, seed=74),
    Case("w_5x5", 2, 17, 39, 68, 5, 5, seed=75),
    Case("w_7x7", 2, 19, 23, 36, 7, 7, seed=76),
    Case("w_1x15", 4, 2, 300, 44, 1, 15, act="normal", seed=77),
    Case("w_1x31", 3, 3, 290, 68, 1, 31, act="normal", seed=78),
    Case("w_many_tiles", 16, 64, 64, 96, 3, 3, seed=79),
    # NCHW, stride 1: the four column phases of the input box, bands, ragged edges
    Case("w_nchw_3x3_same", 3, 37, 44, 20, 3, 3, layout="nchw", seed=81),
    Case("w_nchw_3x3_pl0", 2, 29, 40, 12, 3, 3, padding=(0, 1, 0, 2), layout="nchw", seed=82),
    Case("w_nchw_3x3_pl2", 2, 31, 36, 12, 3, 3, padding=(2, 0, 2, 0), layout="nchw", seed=83),
    Case("w_nchw_3x3_pl3", 2, 26, 40, 12, 3, 3, padding=(1, 3, 3, 3), layout="nchw", seed=84),
    Case("w_nchw_5x5", 2, 35, 52, 10, 5, 5, layout="nchw", seed=85),
    Case("w_nchw_7x7", 2, 33, 28, 9, 7, 7, layout="nchw", seed=86),
    Case("w_nchw_wide", 1, 70, 300, 3, 3, 3, layout="nchw", seed=87),
    Case("w_nchw_planes", 8, 20, 24, 64, 3, 3, layout="nchw", seed=88),
    # NCHW, 1 x kW: rows kernel (channel groups of 8 with a ragged last group)
    Case("w_nchw_1x31", 3, 2, 300, 20, 1, 31, act="normal", layout="nchw", seed=89),
    Case("w_nchw_1x15_pad", 2, 3, 64, 11, 1, 15, padding=(1, 0, 6, 8), act="normal",
         layout="nchw", seed=90),
    Case("w_nchw_1x3", 2, 5, 40, 9, 1, 3, padding=(0, 0, 0, 2), layout="nchw", seed=91),
    Case("w_nchw_1x7", 5, 1, 44, 16, 1, 7, padding=(0, 0, 5, 1), layout="nchw", seed=92),
    # NCHW, stride 2 (3x3): two outputs per lane, the box start's column phases
    Case("w_nchw_s2_pad1", 2, 29, 40, 12, 3, 3, stride=2, padding=1, layout="nchw", seed=93),
    Case("w_nchw_s2_same", 2, 30, 48, 6, 3, 3, stride=2, layout="nchw", seed=94),
    Case("w_nchw_s2_pl3", 1, 26, 44, 5, 3, 3, stride=2, padding=(1, 1, 3, 2), layout="nchw", seed=95),
    Case("w_nchw_s2_pl2", 1, 33, 44, 7, 3, 3, stride=2, padding=(2, 0, 2, 4), layout="nchw", seed=96),
]


@pytest.mark.parametrize("case", TILED, ids=lambda c: c.name)
def test_tiled_weight_gradient(case):
    inp = gu.inputs(case)
    x, dy = inp["x"].cuda(), inp["dy"].cuda()
    dwt = torch.empty(case.C, case.kH, case.kW, device="cuda")
    assert dw.dwconv2d_query_algo(gu.desc_of(case), 2, x.data_ptr(), dy.data_ptr(),
                                  dwt.data_ptr()) == dw.DW_ALGO_TILED
    check(case, algos=("tiled", "direct"))


def test_repeatable_bit_for_bit():
    case = wl.mobilenet()[2]
    inp = gu.inputs(case)
    a = gpu(case, inp)
    b = gpu(case, inp)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_large_full_size(layout):
    case = [c for c in wl.large() if c.H == 512 and c.layout == layout][0]
    check(case, algos=("auto",))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_mobilenet_stride2_full_size(layout):
    case = wl.mobilenet()[2].with_(layout=layout)
    check(case, algos=("auto",))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_conformer_full_size(layout):
    case = [c for c in wl.conformer() if c.W == 512 and c.layout == layout][0]
    check(case, algos=("auto",))


def test_random_sweep():
    rng = np.random.default_rng(303)
    count = 0
    while count < 40:
        layout = "nhwc" if rng.random() < 0.5 else "nchw"
        k = int(rng.choice([1, 2, 3, 5]))
        case = Case(f"wsweep{count}", int(rng.integers(1, 4)), int(rng.integers(1, 30)),
                    int(rng.integers(1, 30)), int(rng.choice([1, 4, 7, 32, 36])), k,
                    int(rng.choice([1, k])), stride=int(rng.integers(1, 3)),
                    dilation=int(rng.integers(1, 3)),
                    padding="same" if rng.random() < 0.5 else int(rng.integers(0, 3)),
                    layout=layout, seed=7000 + count)
        ho, wo = gu.out_hw(case)
        if ho < 1 or wo < 1:
            continue
        check(case)
        count += 1


def test_no_bias_gradient_and_small_workspace_error():
    case = Case("wnob", 2, 12, 12, 32, 3, 3, seed=80)
    inp = gu.inputs(case)
    dwr, _, dws, _ = reference(case, inp)
    g_w, g_b = dw.dwconv2d_bwd_weight(inp["x"].cuda(), inp["dy"].cuda(), (3, 3), bias=False)
    torch.cuda.synchronize()
    assert g_b is None
    gu.assert_close(g_w.cpu().numpy(), dwr, dws, "dW without db")
    with pytest.raises(ValueError):
        dw.dwconv2d_bwd_weight(inp["x"].cuda(), inp["dy"].cuda(), (3, 3),
                               workspace=torch.empty(8, dtype=torch.uint8, device="cuda"))


# NCHW tiled weight gradient with 16-bit activations: every column phase of
# the 16-byte x box (REM 0..3 and the extra 4-element shift), stride 2, 5x5,
# 7x7, a multiplier and the 1 x kW rows kernel; float32 results, the same bits as the float32 call on
# the widened tensors (same kernel family, same summation order)
HALF_NCHW = [
    Case("wh_3x3_same", 2, 37, 48, 6, 3, 3, layout="nchw", seed=91),
    Case("wh_3x3_pl0", 2, 29, 40, 5, 3, 3, padding=(0, 1, 0, 2), layout="nchw", seed=92),
    Case("wh_3x3_pl2", 1, 31, 40, 4, 3, 3, padding=(2, 0, 2, 0), layout="nchw", seed=93),
    Case("wh_3x3_pl3", 1, 26, 40, 6, 3, 3, padding=(1, 3, 3, 7), layout="nchw", seed=94),
    Case("wh_3x3_pl5", 1, 21, 40, 5, 3, 3, padding=(1, 1, 5, 5), layout="nchw", seed=95),
    Case("wh_3x3_pl4", 1, 17, 40, 3, 3, 3, padding=(1, 1, 4, 6), layout="nchw", seed=100),
    Case("wh_3x3_pl6", 1, 17, 40, 3, 3, 3, padding=(1, 1, 6, 4), layout="nchw", seed=101),
    Case("wh_3x3_pl7", 1, 17, 40, 3, 3, 3, padding=(1, 1, 7, 3), layout="nchw", seed=102),
    Case("wh_3x3_s2", 3, 29, 80, 4, 3, 3, stride=2, padding=1, layout="nchw", seed=96),
    Case("wh_5x5", 2, 35, 48, 5, 5, 5, layout="nchw", seed=97),
    Case("wh_7x7", 2, 33, 32, 4, 7, 7, layout="nchw", seed=98),
    Case("wh_m2_3x3", 2, 21, 40, 3, 3, 3, multiplier=2, layout="nchw", seed=99),
    # 1 x kW filters: the rows kernel
    Case("wh_1x31", 3, 2, 296, 10, 1, 31, act="normal", layout="nchw", seed=103),
    Case("wh_1x15_pad", 2, 3, 64, 11, 1, 15, padding=(0, 0, 6, 8), act="normal",
         layout="nchw", seed=104),
    Case("wh_1x7_pl5", 2, 2, 40, 9, 1, 7, padding=(0, 0, 5, 1), layout="nchw", seed=105),
    Case("wh_1x3_pl4", 1, 3, 48, 12, 1, 3, padding=(0, 0, 4, 6), layout="nchw", seed=106),
]


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("case", HALF_NCHW, ids=lambda c: c.name)
def test_nchw_tiled_half_weight_gradient(case, dt):
    inp = gu.inputs(case)
    x16, g16 = inp["x"].to(dt), inp["dy"].to(dt)
    x32, g32 = x16.float(), g16.float()
    p = gu.problem(case)
    xd, gd = gu.f64(x32), gu.f64(g32)
    dwr, dbr = oracle.bwd_weight(p, xd, gd)
    dws, dbs = oracle.bwd_weight(p, np.abs(xd), np.abs(gd))
    desc = gu.desc_of(case)
    desc.atype = dw.DW_F16 if dt == torch.float16 else dw.DW_BF16
    gw = torch.empty(case.multiplier * case.C, case.kH, case.kW, device="cuda")
    xc, gc = x16.cuda(), g16.cuda()
    assert dw.dwconv2d_query_algo(desc, 2, xc.data_ptr(), gc.data_ptr(), gw.data_ptr()) == \
        dw.DW_ALGO_TILED
    kw = dict(stride=case.stride, dilation=case.dilation, padding=case.padding,
              layout=case.layout)
    a_w, a_b = dw.dwconv2d_bwd_weight(xc, gc, (case.kH, case.kW), **kw)
    b_w, b_b = dw.dwconv2d_bwd_weight(x32.cuda(), g32.cuda(), (case.kH, case.kW), **kw)
    d_w, d_b = dw.dwconv2d_bwd_weight(xc, gc, (case.kH, case.kW), algo="direct", **kw)
    torch.cuda.synchronize()
    gu.assert_close(a_w.cpu().numpy(), dwr, dws, f"{case.name} dW")
    gu.assert_close(a_b.cpu().numpy(), dbr, dbs, f"{case.name} db")
    gu.assert_close(d_w.cpu().numpy(), dwr, dws, f"{case.name} dW direct")
    assert torch.equal(a_w, b_w) and torch.equal(a_b, b_b)
