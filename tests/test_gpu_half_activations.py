"""GPU parity with float16 and bfloat16 activations (x, y, dy, dx stored in
16 bits, every sum formed in float32, each result rounded once).

Reference: the float64 oracle on the 16-bit input values.  Rule per
element, from the arithmetic: the float32 result obeys the float32 rule
(|r32 - ref| <= 1e-5 * S, S = sum|terms|), and one rounding to the storage
type adds at most u * |r32| (u = 2^-11 for float16, 2^-8 for bfloat16) plus
half the smallest float16 subnormal, so
    |gpu - ref| <= 1e-5 * S * (1 + u) + u * |ref| + 2^-25.
Bit-level rule: the 16-bit call returns exactly the float32 call's result on
the widened inputs, rounded to nearest even (the same kernel family sums in
the same order), and the weight gradient (float32 outputs) equals the
float32 call's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200 import build as dwbuild
from depthwise_convolution_fwd_b200.workloads import Case
from depthwise_convolution_fwd_b200 import workloads as wl
from tests import gpu_util as gu
from tests import test_gpu_fused_epilogue as fe

pytestmark = pytest.mark.gpu

DTYPES = {"f16": (torch.float16, 2.0 ** -11), "bf16": (torch.bfloat16, 2.0 ** -8)}


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dwbuild.build()
    dw.lib()
    yield
    torch.cuda.synchronize()
    assert dw.dwconv2d_take_device_error() == 0


def inputs16(case, dt):
    inp = dict(gu.inputs(case))
    inp["x"] = inp["x"].to(dt)
    inp["dy"] = inp["dy"].to(dt)
    return inp


def widened(inp):
    out = dict(inp)
    out["x"] = inp["x"].float()
    out["dy"] = inp["dy"].float()
    return out


def check16(got, ref, scale, u, what):
    g = got.float().cpu().numpy().astype(np.float64).reshape(-1)
    r = np.asarray(ref, dtype=np.float64).reshape(-1)
    s = np.asarray(scale, dtype=np.float64).reshape(-1)
    assert np.all(np.isfinite(g)), what
    tol = 1e-5 * s * (1 + u) + u * np.abs(r) + 2.0 ** -25
    bad = np.abs(g - r) > tol
    if bad.any():
        i = int(np.flatnonzero(bad)[0])
        raise AssertionError(f"{what}: |gpu-ref| {abs(g[i] - r[i]):.3e} > {tol[i]:.3e} at {i} "
                             f"(gpu {g[i]!r}, ref {r[i]!r}), {int(bad.sum())} elements")


def run_case(case, name, algo="auto"):
    dt, u = DTYPES[name]
    inp = inputs16(case, dt)
    w32 = widened(inp)
    # forward
    ref, scale = gu.reference_fwd(case, w32)
    y = gu.gpu_fwd(case, inp, algo)
    y32 = gu.gpu_fwd(case, w32, algo)
    torch.cuda.synchronize()
    assert y.dtype == dt
    check16(y, ref, scale, u, f"{case.name} {name} fwd [{algo}]")
    assert torch.equal(y, y32.to(dt)), f"{case.name} {name} fwd is not the rounded float32 result"
    # input gradient
    ref, scale = gu.reference_bwd(case, w32)
    dx = gu.gpu_bwd(case, inp, algo)
    dx32 = gu.gpu_bwd(case, w32, algo)
    torch.cuda.synchronize()
    check16(dx, ref, scale, u, f"{case.name} {name} bwd [{algo}]")
    assert torch.equal(dx, dx32.to(dt)), f"{case.name} {name} bwd is not the rounded float32 result"
    # weight gradient: float32 outputs, the float32 call's bits
    p = gu.problem(case)
    x64, dy64 = gu.f64(w32["x"]), gu.f64(w32["dy"])
    dwr, dbr = oracle.bwd_weight(p, x64, dy64)
    dws, dbs = oracle.bwd_weight(p, np.abs(x64), np.abs(dy64))
    # (the weight gradient has no tiled kernel for some shapes the others cover)
    kw = dict(stride=case.stride, dilation=case.dilation, padding=case.padding,
              layout=case.layout, algo="auto" if algo == "tiled" else algo)
    gw, gb = dw.dwconv2d_bwd_weight(inp["x"].cuda(), inp["dy"].cuda(), (case.kH, case.kW), **kw)
    gw32, gb32 = dw.dwconv2d_bwd_weight(w32["x"].cuda(), w32["dy"].cuda(), (case.kH, case.kW), **kw)
    torch.cuda.synchronize()
    gu.assert_close(gw.cpu().numpy(), dwr, dws, f"{case.name} {name} dW")
    gu.assert_close(gb.cpu().numpy(), dbr, dbs, f"{case.name} {name} db")
    # same bits when both calls run the same kernel family (NCHW weight
    # gradients of 16-bit activations use the direct kernel)
    d16, d32 = gu.desc_of(case, kw["algo"]), gu.desc_of(case, kw["algo"])
    d16.atype = {"f16": dw.DW_F16, "bf16": dw.DW_BF16}[name]
    xp, gp = inp["x"].cuda(), inp["dy"].cuda()
    if (dw.dwconv2d_query_algo(d16, 2, xp.data_ptr(), gp.data_ptr(), gw.data_ptr()) ==
            dw.dwconv2d_query_algo(d32, 2, xp.data_ptr(), gp.data_ptr(), gw.data_ptr())):
        assert torch.equal(gw, gw32) and torch.equal(gb, gb32)


TILED = [
    Case("h_3x3", 2, 37, 45, 72, 3, 3, seed=401),
    Case("h_3x3_big", 4, 64, 64, 128, 3, 3, seed=402),
    Case("h_3x3_s2", 4, 29, 41, 48, 3, 3, stride=2, padding=1, seed=403),
    Case("h_3x3_s2_same", 2, 30, 34, 40, 3, 3, stride=2, seed=404),
    Case("h_3x3_d2", 2, 23, 30, 40, 3, 3, dilation=2, seed=405),
    Case("h_5x5", 2, 17, 39, 72, 5, 5, seed=406),
    Case("h_7x7", 2, 19, 23, 40, 7, 7, seed=407),
    Case("h_1x15", 4, 2, 300, 48, 1, 15, act="normal", seed=408),
    Case("h_1x31", 3, 3, 290, 72, 1, 31, act="normal", seed=409),
]


@pytest.mark.parametrize("name", ["f16", "bf16"])
@pytest.mark.parametrize("case", TILED, ids=lambda c: c.name)
def test_tiled_half_activations(case, name):
    dt, _ = DTYPES[name]
    inp = inputs16(case, dt)
    x = inp["x"].cuda()
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda", dtype=dt)
    desc = gu.desc_of(case)
    desc.atype = {"f16": dw.DW_F16, "bf16": dw.DW_BF16}[name]
    assert dw.dwconv2d_query_algo(desc, 0, x.data_ptr(), inp["w"].cuda().data_ptr(),
                                  y.data_ptr()) == dw.DW_ALGO_TILED
    assert dw.dwconv2d_query_algo(desc, 1, y.data_ptr(), inp["w"].cuda().data_ptr(),
                                  x.data_ptr()) == dw.DW_ALGO_TILED
    run_case(case, name, "tiled")


# NCHW: every column phase of the 16-byte box start (REM 0..3, extra shift 0 or 4)
NCHW = [
    Case("hn_3x3_same", 2, 37, 48, 6, 3, 3, layout="nchw", seed=421),
    Case("hn_3x3_pl0", 2, 29, 40, 5, 3, 3, padding=(0, 1, 0, 2), layout="nchw", seed=422),
    Case("hn_3x3_pl2", 2, 31, 40, 4, 3, 3, padding=(2, 0, 2, 0), layout="nchw", seed=423),
    Case("hn_3x3_pl3", 1, 26, 40, 6, 3, 3, padding=(1, 3, 3, 7), layout="nchw", seed=424),
    Case("hn_3x3_pl5", 1, 21, 40, 5, 3, 3, padding=(1, 1, 5, 5), layout="nchw", seed=425),
    Case("hn_5x5", 2, 35, 48, 5, 5, 5, layout="nchw", seed=426),
    Case("hn_7x7", 2, 33, 32, 4, 7, 7, layout="nchw", seed=427),
    Case("hn_1x31", 2, 2, 296, 40, 1, 31, act="normal", layout="nchw", seed=428),
    Case("hn_1x15_pad", 2, 3, 64, 11, 1, 15, padding=(1, 0, 6, 8), act="normal",
         layout="nchw", seed=429),
    Case("hn_1x31_ragged", 1, 1, 296, 36, 1, 31, padding=(0, 0, 15, 14), act="normal",
         layout="nchw", seed=430),
]


@pytest.mark.parametrize("name", ["f16", "bf16"])
@pytest.mark.parametrize("case", NCHW, ids=lambda c: c.name)
def test_nchw_tiled_half_activations(case, name):
    dt, _ = DTYPES[name]
    inp = inputs16(case, dt)
    x = inp["x"].cuda()
    Ho, Wo = gu.out_hw(case)
    y = torch.empty(case.out_shape(Ho, Wo), device="cuda", dtype=dt)
    desc = gu.desc_of(case)
    desc.atype = {"f16": dw.DW_F16, "bf16": dw.DW_BF16}[name]
    wp = inp["w"].cuda().data_ptr()
    assert dw.dwconv2d_query_algo(desc, 0, x.data_ptr(), wp, y.data_ptr()) == dw.DW_ALGO_TILED
    if Wo % 8 == 0:  # the input gradient reads dy rows of Wo elements
        assert dw.dwconv2d_query_algo(desc, 1, y.data_ptr(), wp, x.data_ptr()) == dw.DW_ALGO_TILED
    run_case(case, name, "auto")


DIRECT = [
    Case("h_nchw_3x3", 2, 13, 16, 6, 3, 3, layout="nchw", seed=411),
    Case("h_nchw_s2", 2, 13, 16, 6, 3, 3, stride=2, layout="nchw", seed=415),
    Case("h_c36", 2, 12, 14, 36, 3, 3, seed=412),   # C % 8 != 0: 16-bit rows not 16-byte
    Case("h_odd", 1, 9, 11, 7, 5, 5, stride=2, dilation=2, seed=413),
    Case("h_nchw_1x31", 2, 1, 70, 8, 1, 31, act="normal", layout="nchw", seed=414),
]


@pytest.mark.parametrize("name", ["f16", "bf16"])
@pytest.mark.parametrize("case", DIRECT + TILED[:3], ids=lambda c: c.name)
def test_direct_half_activations(case, name):
    run_case(case, name, "direct")


@pytest.mark.parametrize("name", ["f16", "bf16"])
def test_fused_epilogue_half(name):
    dt, u = DTYPES[name]
    for case in (TILED[0], TILED[2], DIRECT[0]):
        inp = inputs16(case, dt)
        w32 = widened(inp)
        bn = fe.bn_of(case)
        for act in ("relu6", "silu"):
            ref, tol = fe.bound(case, w32, bn, act)
            y = fe.gpu_fused(case, inp, bn, act)
            y32 = fe.gpu_fused(case, w32, bn, act)
            torch.cuda.synchronize()
            assert y.dtype == dt
            assert torch.equal(y, y32.to(dt)), (case.name, act)
            g = y.float().cpu().numpy().astype(np.float64).reshape(-1)
            assert np.all(np.abs(g - ref) <= tol * (1 + u) + u * np.abs(ref) + 2.0 ** -25), \
                (case.name, act)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("name", ["f16", "bf16"])
def test_full_size_sampled(name, layout):
    dt, u = DTYPES[name]
    rng = np.random.default_rng(31)
    case = [c for c in wl.large() if c.H == 512 and c.layout == layout][0]
    inp = inputs16(case, dt)
    w32 = widened(inp)
    y = gu.gpu_fwd(case, inp)
    dx = gu.gpu_bwd(case, inp)
    torch.cuda.synchronize()
    idx = gu.structured_sample(tuple(y.shape), case.layout, rng, count=4000)
    ref, scale = gu.reference_fwd_at(case, w32, idx)
    check16(y.reshape(-1)[torch.from_numpy(idx).cuda()], ref, scale, u, "large fwd sampled")
    idx = gu.structured_sample(tuple(dx.shape), case.layout, rng, count=4000)
    ref, scale = gu.reference_bwd_at(case, w32, idx)
    check16(dx.reshape(-1)[torch.from_numpy(idx).cuda()], ref, scale, u, "large bwd sampled")
