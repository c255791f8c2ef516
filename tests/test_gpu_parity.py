"""GPU parity: the CUDA kernels (through the C ABI) against the float64 oracle.

Every configuration of the workload set runs forward and input gradient,
elementwise against the oracle under the rule of tests/gpu_util.py
(|gpu - ref| <= 1e-5 * sum|terms|, exact where there are no terms), on both
kernel families where they apply; the full-size large case is checked on a
structured sample of outputs.  float16 weights must give bit-identical
results to float32 weights holding the same (float16-exact) values.
"""
import numpy as np
import pytest
import torch

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


def check_case(case: Case, algos=("auto", "direct")):
    inp = gu.inputs(case)
    ref_y, sc_y = gu.reference_fwd(case, inp)
    ref_dx, sc_dx = gu.reference_bwd(case, inp)
    for algo in algos:
        y = gu.gpu_fwd(case, inp, algo=algo)
        dx = gu.gpu_bwd(case, inp, algo=algo)
        torch.cuda.synchronize()
        gu.assert_close(y.cpu().numpy(), ref_y, sc_y, f"{case.name} fwd [{algo}]")
        gu.assert_close(dx.cpu().numpy(), ref_dx, sc_dx, f"{case.name} bwd_input [{algo}]")
    return inp


SMALL = wl.tiny() + wl.mobilenet() + [c for c in wl.conformer() if c.W == 24] + \
    [c for c in wl.large() if c.H == 30]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_config_cases_match_oracle(case):
    check_case(case)


@pytest.mark.parametrize("case", [c for c in wl.conformer() if c.W == 512], ids=lambda c: c.name)
def test_conformer_long_matches_oracle(case):
    check_case(case, algos=("auto",))


@pytest.mark.parametrize("case", wl.edge(), ids=lambda c: c.name)
def test_edge_cases_match_oracle(case):
    inp = check_case(case)
    if case.wtype == "f16":
        # float16 weights == float32 weights holding the same values, bit for bit
        for algo in ("auto", "direct"):
            y16 = gu.gpu_fwd(case, inp, algo=algo, w_key="w")
            y32 = gu.gpu_fwd(case, inp, algo=algo, w_key="w32")
            d16 = gu.gpu_bwd(case, inp, algo=algo, w_key="w")
            d32 = gu.gpu_bwd(case, inp, algo=algo, w_key="w32")
            assert torch.equal(y16, y32), f"{case.name}: f16/f32 forward differ [{algo}]"
            assert torch.equal(d16, d32), f"{case.name}: f16/f32 input gradient differ [{algo}]"


# Tiled-kernel instances, each forced and compared, with f16 twins.  The NCHW
# cases keep W and Wo multiples of 4 (the TMA row-stride rule applies to the
# input of both directions) and cover every box alignment REM = (-pl) mod 4 of
# the forward and (pl - kW + 1) mod 4 of the input gradient.
TILED = [
    Case("t_nhwc_3x3_s1", 2, 37, 45, 72, 3, 3, seed=1),
    Case("t_nhwc_3x3_s1_pad", 1, 23, 70, 36, 3, 3, padding=(0, 2, 2, 1), seed=2),
    Case("t_nhwc_3x3_s2", 3, 29, 41, 44, 3, 3, stride=2, padding=1, seed=3),
    Case("t_nhwc_3x3_s2_same", 2, 30, 34, 40, 3, 3, stride=2, seed=4),
    Case("t_nhwc_3x3_s2_asym", 2, 19, 23, 8, 3, 3, stride=2, padding=(2, 0, 1, 2), seed=5),
    Case("t_nhwc_3x3_d2", 2, 21, 40, 36, 3, 3, dilation=2, seed=6),
    Case("t_nhwc_3x3_d3", 1, 25, 30, 64, 3, 3, dilation=3, seed=7),
    Case("t_nhwc_5x5", 2, 17, 39, 68, 5, 5, seed=8),
    Case("t_nhwc_5x5_pad", 1, 17, 20, 32, 5, 5, padding=(4, 0, 1, 3), seed=9),
    Case("t_nhwc_1x3", 3, 2, 150, 36, 1, 3, seed=10),
    Case("t_nhwc_1x5", 2, 3, 130, 20, 1, 5, seed=11),
    Case("t_nhwc_1x7", 2, 1, 260, 40, 1, 7, padding=(0, 0, 5, 2), seed=12),
    Case("t_nhwc_1x15", 2, 2, 300, 44, 1, 15, act="normal", seed=13),
    Case("t_nhwc_1x31", 3, 1, 290, 68, 1, 31, act="normal", seed=14),
    Case("t_nhwc_1x31_pad", 1, 1, 100, 32, 1, 31, padding=(1, 2, 31, 0), act="normal", seed=15),
    Case("t_nchw_3x3", 2, 45, 140, 5, 3, 3, layout="nchw", seed=16),
    Case("t_nchw_3x3_pad0", 1, 40, 132, 3, 3, 3, padding=(0, 0, 0, 2), layout="nchw", seed=17),
    Case("t_nchw_3x3_pad2", 1, 40, 132, 3, 3, 3, padding=(2, 1, 2, 0), layout="nchw", seed=18),
    Case("t_nchw_3x3_pad3", 1, 33, 260, 2, 3, 3, padding=(1, 1, 3, 3), layout="nchw", seed=19),
    Case("t_nchw_5x5", 2, 36, 136, 3, 5, 5, layout="nchw", seed=20),
    Case("t_nchw_7x7", 1, 37, 140, 4, 7, 7, layout="nchw", seed=21),
    Case("t_nchw_1x15", 2, 3, 300, 19, 1, 15, layout="nchw", act="normal", seed=22),
    Case("t_nchw_1x31", 2, 2, 264, 21, 1, 31, layout="nchw", act="normal", seed=23),
    Case("t_nchw_1x31_pad", 1, 1, 132, 9, 1, 31, padding=(2, 0, 4, 10), layout="nchw",
         act="normal", seed=24),
]


@pytest.mark.parametrize("case", TILED, ids=lambda c: c.name)
def test_tiled_kernels_match_oracle(case):
    inp = gu.inputs(case)
    x = inp["x"].cuda()
    w = inp["w"].cuda()
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    assert gu.chosen_algo(case, 0, x, w, y) == dw.DW_ALGO_TILED, "expected the tiled path"
    assert gu.chosen_algo(case, 1, y, w, x) == dw.DW_ALGO_TILED, "expected the tiled path"
    check_case(case, algos=("tiled", "direct"))
    case16 = case.with_(wtype="f16", name=case.name + "_f16")
    inp16 = gu.inputs(case16)
    for fn in (gu.gpu_fwd, gu.gpu_bwd):
        a = fn(case16, inp16, algo="tiled", w_key="w")
        b = fn(case16, inp16, algo="tiled", w_key="w32")
        assert torch.equal(a, b), f"{case.name}: f16 weights not bit-identical"


# Enough tiles that every persistent CTA walks its TMA stage ring several
# times (stage pitch, phase parity and re-issue paths), ragged at every edge.
RING = [
    Case("r_nhwc_3x3_s1", 4, 125, 250, 60, 3, 3, seed=51),
    Case("r_nhwc_3x3_s2", 16, 63, 126, 68, 3, 3, stride=2, padding=1, seed=52),
    Case("r_nhwc_5x5", 16, 61, 125, 64, 5, 5, seed=53),
    Case("r_nhwc_1x31", 16, 15, 250, 124, 1, 31, act="normal", seed=54),
    Case("r_nchw_3x3", 2, 125, 508, 64, 3, 3, layout="nchw", seed=55),
    Case("r_nchw_5x5", 2, 93, 252, 32, 5, 5, layout="nchw", seed=56),
    Case("r_nchw_7x7", 2, 61, 252, 48, 7, 7, layout="nchw", seed=57),
    Case("r_nchw_1x31", 8, 15, 252, 124, 1, 31, layout="nchw", act="normal", seed=58),
]


@pytest.mark.parametrize("case", RING, ids=lambda c: c.name)
def test_tiled_ring_wraps(case):
    inp = gu.inputs(case)
    x = inp["x"].cuda()
    w = inp["w"].cuda()
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    assert gu.chosen_algo(case, 0, x, w, y) == dw.DW_ALGO_TILED
    assert gu.chosen_algo(case, 1, y, w, x) == dw.DW_ALGO_TILED
    check_case(case, algos=("tiled",))


def test_random_sweep_matches_oracle():
    rng = np.random.default_rng(2024)
    count = 0
    while count < 120:
        layout = "nhwc" if rng.random() < 0.5 else "nchw"
        k = int(rng.choice([1, 2, 3, 4, 5, 7, 15, 31]))
        kH, kW = (1, k) if rng.random() < 0.3 else (k, int(rng.choice([1, 3, 5, k])))
        C = int(rng.choice([1, 3, 4, 7, 8, 36, 131, 132]))
        s = int(rng.integers(1, 4))
        d = int(rng.integers(1, 4))
        pad = "same" if rng.random() < 0.5 else tuple(int(v) for v in rng.integers(0, 4, size=4))
        case = Case(f"sweep{count}", int(rng.integers(1, 4)), int(rng.integers(1, 38)),
                    int(rng.integers(1, 38)), C, kH, kW, stride=s, dilation=d, padding=pad,
                    layout=layout, wtype="f16" if rng.random() < 0.3 else "f32",
                    bias=bool(rng.random() < 0.8), seed=5000 + count)
        try:
            ho, wo = gu.out_hw(case)
        except Exception:
            continue
        if ho < 1 or wo < 1:
            continue
        check_case(case)
        count += 1


# ----------------------------------------------------------- full size ---

@pytest.mark.parametrize("case", [c for c in wl.large() if c.H == 512], ids=lambda c: c.name)
def test_large_full_size_sampled(case):
    """1x512x512x256 3x3 SAME, the launch configuration the benchmark times,
    checked on border rows/columns plus 20k random outputs."""
    inp = gu.inputs(case)
    rng = np.random.default_rng(77)
    x = inp["x"].cuda()
    w = inp["w"].cuda()
    b = inp["b"].cuda()
    y = dw.dwconv2d_fwd(x, w, b, padding="same", layout=case.layout)
    assert gu.chosen_algo(case, 0, x, w, y) == dw.DW_ALGO_TILED
    dx = gu.gpu_bwd(case, inp)
    torch.cuda.synchronize()
    iy = gu.structured_sample(tuple(y.shape), case.layout, rng)
    ref, sc = gu.reference_fwd_at(case, inp, iy)
    gu.assert_close(y.reshape(-1).cpu().numpy()[iy], ref, sc, case.name + " fwd")
    ix = gu.structured_sample(tuple(dx.shape), case.layout, rng)
    ref, sc = gu.reference_bwd_at(case, inp, ix)
    gu.assert_close(dx.reshape(-1).cpu().numpy()[ix], ref, sc, case.name + " bwd_input")


# --------------------------------------------------------- memory hygiene --

GUARD = 4096


@pytest.mark.parametrize("case", [
    Case("g_nhwc", 2, 19, 37, 40, 3, 3, seed=31),
    Case("g_nhwc_s2", 2, 19, 37, 44, 3, 3, stride=2, padding=1, seed=32),
    Case("g_nchw", 2, 19, 36, 5, 3, 3, layout="nchw", seed=33),
    Case("g_nhwc_1x31", 2, 1, 70, 36, 1, 31, seed=34),
    Case("g_odd", 2, 9, 11, 7, 5, 5, stride=2, seed=35),
], ids=lambda c: c.name)
@pytest.mark.parametrize("shift", [0, 1])
def test_outputs_stay_inside_their_buffer(case, shift):
    """Canary floats around the output: no kernel writes outside it.  shift=1
    offsets every pointer by one float (unaligned -> direct kernel)."""
    inp = gu.inputs(case)
    canary = float("nan")

    def padded(t):
        buf = torch.full((t.numel() + 2 * GUARD + shift,), 7.0, device="cuda")
        view = buf[GUARD + shift: GUARD + shift + t.numel()].view(t.shape)
        view.copy_(t)
        return buf, view

    _, x = padded(inp["x"])
    _, dy = padded(inp["dy"])
    w = inp["w"].cuda()
    b = inp["b"].cuda()
    ho, wo = gu.out_hw(case)
    for op in ("fwd", "bwd"):
        shape = case.out_shape(ho, wo) if op == "fwd" else case.in_shape()
        n = int(np.prod(shape))
        obuf = torch.full((n + 2 * GUARD + shift,), canary, device="cuda")
        out = obuf[GUARD + shift: GUARD + shift + n].view(shape)
        if op == "fwd":
            dw.dwconv2d_fwd(x, w, b, stride=case.stride, padding=case.padding,
                            layout=case.layout, out=out)
            ref, sc = gu.reference_fwd(case, inp)
        else:
            dw.dwconv2d_bwd_input(dy, w, (case.H, case.W), stride=case.stride,
                                  padding=case.padding, layout=case.layout, out=out)
            ref, sc = gu.reference_bwd(case, inp)
        torch.cuda.synchronize()
        host = obuf.cpu()
        assert torch.isnan(host[:GUARD + shift]).all(), f"{case.name} {op}: write before buffer"
        assert torch.isnan(host[GUARD + shift + n:]).all(), f"{case.name} {op}: write after buffer"
        gu.assert_close(out.cpu().numpy(), ref, sc, f"{case.name} {op} shift={shift}")


def test_input_gradient_overwrites_stale_output():
    case = Case("stale", 2, 16, 20, 8, 3, 3, stride=2, padding=1, seed=41)
    inp = gu.inputs(case)
    ref, sc = gu.reference_bwd(case, inp)
    for algo in ("auto", "direct"):
        out = torch.full(case.in_shape(), 123.0, device="cuda")
        gu.gpu_bwd(case, inp, algo=algo, out=out)
        torch.cuda.synchronize()
        gu.assert_close(out.cpu().numpy(), ref, sc, f"stale [{algo}]")


def test_side_stream_and_repeatability():
    case = wl.mobilenet()[2]
    inp = gu.inputs(case)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y1 = gu.gpu_fwd(case, inp)
        d1 = gu.gpu_bwd(case, inp)
    s.synchronize()
    y2 = gu.gpu_fwd(case, inp)
    d2 = gu.gpu_bwd(case, inp)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(d1, d2)
    ref, sc = gu.reference_fwd(case, inp)
    gu.assert_close(y1.cpu().numpy(), ref, sc, "side stream fwd")


def test_no_bias_and_aliasing_errors_on_device():
    case = Case("nob", 1, 12, 12, 16, 3, 3, bias=False, seed=42)
    inp = gu.inputs(case)
    ref, sc = gu.reference_fwd(case, inp)
    y = gu.gpu_fwd(case, inp)
    torch.cuda.synchronize()
    gu.assert_close(y.cpu().numpy(), ref, sc, "no bias")
    x = inp["x"].cuda()
    with pytest.raises(dw.DwError) as e:
        dw.dwconv2d_fwd(x, inp["w"].cuda(), out=x)
    assert e.value.status == dw.DW_ERR_ALIAS


# ------------------------------------------------- stream-order semantics --

@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("graph", [False, True])
def test_dependent_calls_keep_stream_order(layout, graph):
    """Kernels start early (programmatic dependent launch) but must not touch
    memory before their predecessor on the stream has finished: a chain of
    calls, each reading the previous call's output (tiled and direct kernels
    alternating), must equal the oracle's composition."""
    import oracle
    N, H, W, C = 2, 40, 132, 64
    shape = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
    g = torch.Generator().manual_seed(99)
    x = torch.rand(shape, generator=g) * 2 - 1
    w3 = torch.randn(C, 3, 3, generator=g) / 3
    w5 = torch.randn(C, 5, 5, generator=g) / 5
    b = torch.rand(C, generator=g) * 0.2 - 0.1
    xd, w3d, w5d, bd = x.cuda(), w3.cuda(), w5.cuda(), b.cuda()
    stages = [("fwd", w3d, "tiled"), ("bwd", w5d, "direct"), ("fwd", w5d, "auto"),
              ("bwd", w3d, "tiled"), ("fwd", w3d, "direct"), ("bwd", w3d, "auto")]

    def chain(src):
        t = src
        for op, w, algo in stages:
            if op == "fwd":
                t = dw.dwconv2d_fwd(t, w, bd, layout=layout, algo=algo)
            else:
                t = dw.dwconv2d_bwd_input(t, w, (H, W), layout=layout, algo=algo)
        return t

    if graph:
        chain(xd)  # warm-up outside capture
        torch.cuda.synchronize()
        static_in = xd.clone()
        gr = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        with torch.cuda.graph(gr, stream=s):
            out = chain(static_in)
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        got = out
    else:
        for _ in range(3):
            got = chain(xd)
        torch.cuda.synchronize()

    p3 = oracle.problem(shape, 3, 3, 1, 1, "same", layout)
    p5 = oracle.problem(shape, 5, 5, 1, 1, "same", layout)
    ref = x.double().numpy()
    wmap = {id(w3d): (p3, w3.double().numpy()), id(w5d): (p5, w5.double().numpy())}
    for op, w, _ in stages:
        p, wn = wmap[id(w)]
        ref = oracle.fwd(p, ref, wn, b.double().numpy()) if op == "fwd" else \
            oracle.bwd_input(p, ref, wn)
    err = np.abs(got.cpu().double().numpy() - ref)
    # six chained float32 passes: compare relative to the reference's scale
    assert err.max() <= 1e-4 * np.abs(ref).max(), err.max()


@pytest.mark.parametrize("case", [
    Case("rw_nchw_1x31", 3, 2, 132, 40, 1, 31, padding=(0, 0, 3, 2), layout="nchw",
         act="normal", seed=61),
    Case("rw_nchw_1x15", 2, 3, 260, 36, 1, 15, padding=(1, 0, 0, 1), layout="nchw",
         act="normal", seed=62),
    Case("rw_nchw_3x3", 2, 33, 132, 6, 3, 3, padding=(1, 1, 1, 0), layout="nchw", seed=63),
], ids=lambda c: c.name)
def test_tiled_forward_with_ragged_output_width(case):
    """Forward on the tiled path where the output row pitch is not a
    multiple of 16 bytes (the epilogue falls back to register stores)."""
    inp = gu.inputs(case)
    x = inp["x"].cuda()
    w = inp["w"].cuda()
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    assert gu.out_hw(case)[1] % 4 != 0
    assert gu.chosen_algo(case, 0, x, w, y) == dw.DW_ALGO_TILED
    ref, sc = gu.reference_fwd(case, inp)
    got = gu.gpu_fwd(case, inp, algo="tiled")
    torch.cuda.synchronize()
    gu.assert_close(got.cpu().numpy(), ref, sc, case.name)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("graph", [False, True])
def test_dependent_calls_with_epilogue_and_gradients(layout, graph):
    """Stream order across the other calls: the fused forward's output is the
    next call's dy, whose weight gradient (two kernels and a workspace) and
    input gradient follow, then a forward of that input gradient; eager and
    in a CUDA graph, checked against the oracle's composition."""
    import oracle
    from depthwise_convolution_fwd_b200.workloads import make_bn
    N, H, W, C = 2, 36, 64, 32
    shape = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
    g = torch.Generator().manual_seed(123)
    x = torch.rand(shape, generator=g) * 2 - 1
    w = torch.randn(C, 3, 3, generator=g) / 3
    b = torch.rand(C, generator=g) * 0.2 - 0.1
    bn = make_bn(C, 124)
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    bnd = tuple(t.cuda() for t in bn[:4]) + (bn[4],)
    need = dw.dwconv2d_bwd_weight_workspace_size(dw.make_desc(N, H, W, C, 3, 3, layout=layout))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    gw = torch.empty(C, 3, 3, device="cuda")
    gb = torch.empty(C, device="cuda")

    def chain(src):
        y = dw.dwconv2d_fwd_bn_act(src, wd, bd, bnd, "silu", layout=layout)
        dw.dwconv2d_bwd_weight(src, y, (3, 3), layout=layout, dw=gw, db=gb, workspace=ws)
        dx = dw.dwconv2d_bwd_input(y, wd, (H, W), layout=layout)
        return dw.dwconv2d_fwd(dx, wd, bd, layout=layout), y

    if graph:
        chain(xd)
        torch.cuda.synchronize()
        static_in = xd.clone()
        gr = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        with torch.cuda.graph(gr, stream=s):
            out, y = chain(static_in)
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
    else:
        for _ in range(3):
            out, y = chain(xd)
        torch.cuda.synchronize()

    p = oracle.problem(shape, 3, 3, 1, 1, "same", layout)
    xn, wn, bn_ = x.double().numpy(), w.double().numpy(), b.double().numpy()
    bn64 = tuple(t.double().numpy() for t in bn[:4]) + (bn[4],)
    y_ref = oracle.fwd_bn_act(p, xn, wn, bn_, bn64, "silu")
    assert np.abs(y.cpu().double().numpy() - y_ref).max() <= 1e-4 * np.abs(y_ref).max()
    # the gradients of what the GPU actually produced as y
    yn = y.cpu().double().numpy()
    dw_ref, db_ref = oracle.bwd_weight(p, xn, yn)
    assert np.abs(gw.cpu().double().numpy() - dw_ref).max() <= 1e-4 * np.abs(dw_ref).max()
    assert np.abs(gb.cpu().double().numpy() - db_ref).max() <= 1e-4 * np.abs(db_ref).max()
    out_ref = oracle.fwd(p, oracle.bwd_input(p, yn, wn), wn, bn_)
    assert np.abs(out.cpu().double().numpy() - out_ref).max() <= 1e-4 * np.abs(out_ref).max()
