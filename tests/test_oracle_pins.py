"""Pins of the float64 oracle to facts outside itself (CPU only).

Every check here comes from something other than the oracle's own code:
hand-derived values (tests/golden/), library routines (torch.nn.functional
conv2d and autograd, in float64), identities stated on the source page
("LeanMlir Proofs/Architectures/Depthwise": equality with a grouped conv of
feature_group_count = C, the direct and reversed-kernel input-gradient
formulas, the affine / adjoint structure of the input-VJP, stride 2 as even
or odd decimation of stride-1 SAME), and closed forms (constant input,
impulse, 1x1 kernel, separable kernel).  A dropped term, a wrong sign or
index, a transposed operand or a flipped kernel fails at least one of them.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def prob1(H, W, C, kH, kW, stride, dilation, pads, N=1, layout="nhwc"):
    shape = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
    return oracle.problem(shape, kH, kW, stride, dilation, tuple(pads), layout)


def chw_to(layout, a):
    """(C,H,W) array -> (1,H,W,C) or (1,C,H,W)."""
    a = np.asarray(a, dtype=np.float64)
    return a.transpose(1, 2, 0)[None] if layout == "nhwc" else a[None]


def to_chw(layout, a):
    return a[0].transpose(2, 0, 1) if layout == "nhwc" else a[0]


# ---------------------------------------------------------------- golden ---

@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_golden_orientation(oracle_mod, layout):
    g = load_golden("orientation_2x2.json")
    p = prob1(g["H"], g["W"], 1, g["kH"], g["kW"], g["stride"], g["dilation"],
              g["pads"], layout=layout)
    x = chw_to(layout, [g["x"]])
    w = np.array(g["w"], dtype=np.float64)[None]
    y = oracle.fwd(p, x, w, [g["b"]])
    assert np.array_equal(to_chw(layout, y)[0], np.array(g["y"]))
    for case in g["bwd"]:
        dx = oracle.bwd_input(p, chw_to(layout, [case["dy"]]), w)
        assert np.array_equal(to_chw(layout, dx)[0], np.array(case["dx"]))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_golden_stride2_even_and_odd_decimation(oracle_mod, layout):
    g = load_golden("stride2_4x4.json")
    x = chw_to(layout, [g["x"]])
    w = np.array(g["w"], dtype=np.float64)[None]
    p1 = prob1(4, 4, 1, 3, 3, 1, 1, (1, 1, 1, 1), layout=layout)
    assert np.array_equal(to_chw(layout, oracle.fwd(p1, x, w))[0], np.array(g["same_s1"]))
    # "same" at stride 1 resolves to the same pads
    ps = oracle.problem(x.shape, 3, 3, 1, 1, "same", layout)
    assert list(ps[10:14]) == [1, 1, 1, 1]
    for key in ("even", "xla_same"):
        case = g[key]
        p = prob1(4, 4, 1, 3, 3, case["stride"], 1, case["pads"], layout=layout)
        y = to_chw(layout, oracle.fwd(p, x, w))[0]
        assert np.array_equal(y, np.array(case["y"])), key
        dx = to_chw(layout, oracle.bwd_input(p, chw_to(layout, [case["dy"]]), w))[0]
        assert np.array_equal(dx, np.array(case["dx"])), key
    # the "same" mode at stride 2 is the XLA rule -> odd decimation
    px = oracle.problem(x.shape, 3, 3, 2, 1, "same", layout)
    assert list(px[10:14]) == g["xla_same"]["pads"]


def test_golden_dilation(oracle_mod):
    g = load_golden("dilation2_5x5.json")
    p = prob1(5, 5, 1, 2, 2, g["stride"], g["dilation"], g["pads"])
    y = oracle.fwd(p, chw_to("nhwc", [g["x"]]), np.array(g["w"], float)[None])
    assert np.array_equal(to_chw("nhwc", y)[0], np.array(g["y"]))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_golden_channels_and_asymmetric_pads(oracle_mod, layout):
    g = load_golden("channels_2ch.json")
    p = prob1(2, 2, 2, 2, 2, g["stride"], g["dilation"], g["pads"], layout=layout)
    y = oracle.fwd(p, chw_to(layout, g["x"]), np.array(g["w"], float), g["b"])
    assert np.array_equal(to_chw(layout, y), np.array(g["y"]))


def test_golden_shape_pins(oracle_mod):
    g = load_golden("shape_pins.json")
    for e in g["extent"]:
        assert oracle.out_extent(e["in"], e["k"], e["s"], e["d"], e["lo"], e["hi"]) == e["out"], e
    for e in g["same"]:
        assert oracle.same_pads(e["in"], e["k"], e["s"], e["d"]) == (e["lo"], e["hi"]), e
    # the issue's forward: 1x4x4x4 (N,C,H,W) with a 3x3 kernel, groups = 4, no pad
    p = oracle.problem((1, 4, 4, 4), 3, 3, 1, 1, 0, "nchw")
    assert oracle.out_shape(p) == (1, 4, 2, 2)


# ---------------------------------------------------- library routines ----

def random_case(rng, layout=None, max_hw=9, max_k=4, max_c=3, max_n=2):
    layout = layout or rng.choice(["nhwc", "nchw"])
    N = int(rng.integers(1, max_n + 1))
    C = int(rng.integers(1, max_c + 1))
    H = int(rng.integers(1, max_hw + 1))
    W = int(rng.integers(1, max_hw + 1))
    kH = int(rng.integers(1, max_k + 1))
    kW = int(rng.integers(1, max_k + 1))
    sh, sw = (int(v) for v in rng.integers(1, 4, size=2))
    dh, dw = (int(v) for v in rng.integers(1, 4, size=2))
    if rng.random() < 0.3:
        pads = "same"
    else:
        pads = tuple(int(v) for v in rng.integers(0, 4, size=4))
    shape = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
    p = oracle.problem(shape, kH, kW, (sh, sw), (dh, dw), pads, layout)
    return p, layout


def valid_cases(seed, count, **kw):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < count:
        p, layout = random_case(rng, **kw)
        if min(oracle.out_shape(p)) > 0:
            out.append((p, layout, rng))
    return out


def to_nchw(p, a):
    return a.transpose(0, 3, 1, 2) if int(p[14]) == 0 else a


def from_nchw(p, a):
    return a.transpose(0, 2, 3, 1) if int(p[14]) == 0 else a


def torch_fwd(p, x, w, b, dense=False):
    """Library routine: torch conv2d in float64 on an explicitly padded input."""
    N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr, _, M = (int(v) for v in p)
    xt = torch.from_numpy(np.ascontiguousarray(to_nchw(p, x)))
    xt = F.pad(xt, (pl, pr, pt, pb))
    wt = torch.from_numpy(np.asarray(w, dtype=np.float64).reshape(C * M, 1, kH, kW))
    if dense:
        # dense kernel Wd[o,i] = delta_{i, o // M} W[o]: a regular conv
        wd = torch.zeros(C * M, C, kH, kW, dtype=torch.float64)
        for o in range(C * M):
            wd[o, o // M] = wt[o, 0]
        y = F.conv2d(xt, wd, None, (sh, sw), 0, (dh, dw), groups=1)
    else:
        y = F.conv2d(xt, wt, None, (sh, sw), 0, (dh, dw), groups=C)
    if b is not None:
        y = y + torch.from_numpy(np.asarray(b, dtype=np.float64)).view(1, C * M, 1, 1)
    return from_nchw(p, y.numpy())


@pytest.mark.parametrize("dense", [False, True])
def test_fwd_equals_torch_conv2d(oracle_mod, dense):
    for p, layout, rng in valid_cases(11 + dense, 60):
        x = rng.standard_normal(oracle.in_shape(p))
        w = rng.standard_normal((int(p[3]), int(p[4]), int(p[5])))
        b = rng.standard_normal(int(p[3]))
        y = oracle.fwd(p, x, w, b)
        ref = torch_fwd(p, x, w, b, dense=dense)
        assert y.shape == ref.shape
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_bwd_equals_torch_autograd(oracle_mod):
    for p, layout, rng in valid_cases(21, 60):
        x = rng.standard_normal(oracle.in_shape(p))
        w = rng.standard_normal((int(p[3]), int(p[4]), int(p[5])))
        dy = rng.standard_normal(oracle.out_shape(p))
        xt = torch.from_numpy(x).requires_grad_(True)
        N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr, _, _ = (int(v) for v in p)
        xn = xt.permute(0, 3, 1, 2) if layout == "nhwc" else xt
        yt = F.conv2d(F.pad(xn, (pl, pr, pt, pb)),
                      torch.from_numpy(w).view(C, 1, kH, kW), None,
                      (sh, sw), 0, (dh, dw), groups=C)
        dyt = torch.from_numpy(np.ascontiguousarray(to_nchw(p, dy)))
        (gx,) = torch.autograd.grad(yt, xt, dyt)
        np.testing.assert_allclose(oracle.bwd_input(p, dy, w), gx.numpy(),
                                   rtol=1e-12, atol=1e-12)


# ------------------------------------------------ identities of the page --

def grouped_conv_bruteforce(x, wg, groups, stride, dilation, pads):
    """Generic grouped conv (NCHW, one image) with feature_group_count = groups,
    written out with an explicit sum over the input channels of each group."""
    C_in, H, W = x.shape
    C_out, cpg, kH, kW = wg.shape
    sh, sw = stride
    dh, dw = dilation
    pt, pb, pl, pr = pads
    Ho = (H + pt + pb - dh * (kH - 1) - 1) // sh + 1
    Wo = (W + pl + pr - dw * (kW - 1) - 1) // sw + 1
    opg = C_out // groups
    y = np.zeros((C_out, Ho, Wo))
    for o in range(C_out):
        g = o // opg
        for ho in range(Ho):
            for wo in range(Wo):
                s = 0.0
                for ci in range(cpg):
                    i = g * cpg + ci
                    for kh in range(kH):
                        for kw in range(kW):
                            hh = ho * sh + kh * dh - pt
                            ww = wo * sw + kw * dw - pl
                            if 0 <= hh < H and 0 <= ww < W:
                                s += x[i, hh, ww] * wg[o, ci, kh, kw]
                y[o, ho, wo] = s
    return y


def test_fwd_equals_block_diagonal_dense_conv_bruteforce(oracle_mod):
    """Depthwise == a regular conv (groups = 1) whose kernel is block-diagonal,
    == a grouped conv with feature_group_count = C."""
    for p, layout, rng in valid_cases(31, 25, max_hw=6, max_k=3, max_c=3, max_n=1):
        N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr, _, _ = (int(v) for v in p)
        x = rng.standard_normal(oracle.in_shape(p))
        w = rng.standard_normal((C, kH, kW))
        xc = to_nchw(p, x)[0]
        wd = np.zeros((C, C, kH, kW))
        for c in range(C):
            wd[c, c] = w[c]
        dense = grouped_conv_bruteforce(xc, wd, 1, (sh, sw), (dh, dw), (pt, pb, pl, pr))
        grouped = grouped_conv_bruteforce(xc, w[:, None], C, (sh, sw), (dh, dw), (pt, pb, pl, pr))
        y = to_nchw(p, oracle.fwd(p, x, w))[0]
        np.testing.assert_allclose(y, dense, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(y, grouped, rtol=1e-12, atol=1e-12)


def bwd_direct_formula_full(p, dy, w):
    """The page's closed-form input gradient: for each input position a sum
    over ALL output positions (ho,wo), with the kernel offset reconstructed
    from hi + pt = ho*sh + kh*dh; a term counts only when that offset is a
    whole tap in [0,kH) x [0,kW)."""
    N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr, _, _ = (int(v) for v in p)
    dyc = to_nchw(p, dy)
    Ho, Wo = dyc.shape[2], dyc.shape[3]
    dx = np.zeros((N, C, H, W))
    for n, c, hi, wi in itertools.product(range(N), range(C), range(H), range(W)):
        s = 0.0
        for ho in range(Ho):
            for wo in range(Wo):
                a, bb = hi + pt - ho * sh, wi + pl - wo * sw
                if a % dh or bb % dw:
                    continue
                kh, kw = a // dh, bb // dw
                if 0 <= kh < kH and 0 <= kw < kW:
                    s += w[c, kh, kw] * dyc[n, c, ho, wo]
        dx[n, c, hi, wi] = s
    return from_nchw(p, dx)


def test_bwd_equals_direct_formula(oracle_mod):
    for p, layout, rng in valid_cases(41, 40, max_hw=7):
        w = rng.standard_normal((int(p[3]), int(p[4]), int(p[5])))
        dy = rng.standard_normal(oracle.out_shape(p))
        ref = bwd_direct_formula_full(p, dy, w)
        np.testing.assert_allclose(oracle.bwd_input(p, dy, w), ref, rtol=1e-12, atol=1e-12)


def test_bwd_equals_reversed_kernel_formula_stride1(oracle_mod):
    """Stride 1: dx[c,h,w] = sum W[c,kH-1-kh,kW-1-kw] dy[c, h+kh*d-p't, w+kw*d-p'l]
    with p' = d(k-1) - p_lo (the page's formula uses the forward's p, which
    coincides for symmetric pads)."""
    rng = np.random.default_rng(51)
    count = 0
    while count < 40:
        p, layout = random_case(rng)
        p[6] = p[7] = 1
        if min(oracle.out_shape(p)) <= 0:
            continue
        count += 1
        N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr, _, _ = (int(v) for v in p)
        w = rng.standard_normal((C, kH, kW))
        dy = rng.standard_normal(oracle.out_shape(p))
        dyc = to_nchw(p, dy)
        Ho, Wo = dyc.shape[2:]
        ppt, ppl = dh * (kH - 1) - pt, dw * (kW - 1) - pl
        dx = np.zeros((N, C, H, W))
        for n, c, h, ww in itertools.product(range(N), range(C), range(H), range(W)):
            s = 0.0
            for kh in range(kH):
                for kw in range(kW):
                    r, q = h + kh * dh - ppt, ww + kw * dw - ppl
                    if 0 <= r < Ho and 0 <= q < Wo:
                        s += w[c, kH - 1 - kh, kW - 1 - kw] * dyc[n, c, r, q]
            dx[n, c, h, ww] = s
        np.testing.assert_allclose(oracle.bwd_input(p, dy, w), from_nchw(p, dx),
                                   rtol=1e-12, atol=1e-12)


def test_adjoint_identity(oracle_mod):
    """<dy, J x> = <J^T dy, x> with J the forward at b = 0."""
    for p, layout, rng in valid_cases(61, 80, max_hw=12, max_k=5, max_c=4, max_n=2):
        x = rng.standard_normal(oracle.in_shape(p))
        w = rng.standard_normal((int(p[3]), int(p[4]), int(p[5])))
        dy = rng.standard_normal(oracle.out_shape(p))
        lhs = float(np.sum(dy * oracle.fwd(p, x, w)))
        rhs = float(np.sum(oracle.bwd_input(p, dy, w) * x))
        assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), (lhs, rhs)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("k", [1, 3, 5, 7])
def test_stride2_is_decimation_of_stride1_same(oracle_mod, layout, k):
    """Stride-2 with symmetric pad (k-1)/2 keeps the even positions of the
    stride-1 SAME output; the XLA SAME rule at stride 2 keeps the odd ones
    (even input extents, odd k >= 3; at k = 1 the rule pads nothing and keeps
    the even ones).  The strided input-VJP zero-upsamples dy onto
    those positions and runs the stride-1 input-VJP."""
    rng = np.random.default_rng(71 + k)
    for (H, W, C, N) in [(8, 6, 3, 2), (4, 10, 2, 1), (6, 6, 1, 1)]:
        shape = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
        x = rng.standard_normal(shape)
        w = rng.standard_normal((C, k, k))
        b = rng.standard_normal(C)
        p1 = oracle.problem(shape, k, k, 1, 1, "same", layout)
        y1 = to_nchw(p1, oracle.fwd(p1, x, w, b))
        half = (k - 1) // 2
        pe = oracle.problem(shape, k, k, 2, 1, half, layout)
        po = oracle.problem(shape, k, k, 2, 1, "same", layout)
        ye = to_nchw(pe, oracle.fwd(pe, x, w, b))
        yo = to_nchw(po, oracle.fwd(po, x, w, b))
        np.testing.assert_allclose(ye, y1[:, :, 0::2, 0::2], rtol=1e-13, atol=1e-13)
        odd = 1 if k > 1 else 0
        np.testing.assert_allclose(yo, y1[:, :, odd::2, odd::2], rtol=1e-13, atol=1e-13)
        for p2, phase in ((pe, 0), (po, odd)):
            dy2 = rng.standard_normal(oracle.out_shape(p2))
            up = np.zeros(to_nchw(p1, np.zeros(oracle.out_shape(p1))).shape)
            up[:, :, phase::2, phase::2] = to_nchw(p2, dy2)
            ref = oracle.bwd_input(p1, from_nchw(p1, up), w)
            np.testing.assert_allclose(oracle.bwd_input(p2, dy2, w), ref,
                                       rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_constant_input(oracle_mod, layout):
    """x == a: interior outputs = a * sum(W) + b; SAME 3x3 corner = a * (sum of
    the four taps that stay inside) + b."""
    rng = np.random.default_rng(81)
    N, H, W, C = 2, 7, 9, 5
    shape = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
    a = 1.75
    x = np.full(shape, a)
    w = rng.standard_normal((C, 3, 3))
    b = rng.standard_normal(C)
    p = oracle.problem(shape, 3, 3, 1, 1, "same", layout)
    y = to_nchw(p, oracle.fwd(p, x, w, b))
    for c in range(C):
        interior = a * w[c].sum() + b[c]
        np.testing.assert_allclose(y[:, c, 1:-1, 1:-1], interior, rtol=1e-14)
        np.testing.assert_allclose(y[:, c, 0, 0], a * w[c, 1:, 1:].sum() + b[c], rtol=1e-14)
        np.testing.assert_allclose(y[:, c, -1, -1], a * w[c, :2, :2].sum() + b[c], rtol=1e-14)
        np.testing.assert_allclose(y[:, c, 0, 4], a * w[c, 1:, :].sum() + b[c], rtol=1e-14)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_impulse_orientation(oracle_mod, layout):
    """x = delta at (h0,w0): y[h0 - kh*d + pt, w0 - kw*d + pl] = W[kh,kw] + b
    (unflipped); dy = delta at (ho,wo): dx[ho + kh*d - pt, wo + kw*d - pl] = W[kh,kw]."""
    rng = np.random.default_rng(91)
    H, W, C, kH, kW, d = 11, 12, 2, 3, 4, 2
    pt, pb, pl, pr = 3, 2, 4, 1
    shape = (1, H, W, C) if layout == "nhwc" else (1, C, H, W)
    p = oracle.problem(shape, kH, kW, 1, d, (pt, pb, pl, pr), layout)
    w = rng.standard_normal((C, kH, kW))
    b = rng.standard_normal(C)
    h0, w0 = 6, 7
    x = np.zeros((C, H, W))
    x[:, h0, w0] = 1.0
    y = to_nchw(p, oracle.fwd(p, chw_to(layout, x), w, b))[0]
    Ho, Wo = y.shape[1:]
    expect = np.broadcast_to(b[:, None, None], y.shape).copy()
    for kh in range(kH):
        for kw in range(kW):
            ho, wo = h0 - kh * d + pt, w0 - kw * d + pl
            if 0 <= ho < Ho and 0 <= wo < Wo:
                expect[:, ho, wo] += w[:, kh, kw]
    np.testing.assert_array_equal(y, expect)
    ho, wo = 4, 5
    dy = np.zeros((C, Ho, Wo))
    dy[:, ho, wo] = 1.0
    dx = to_nchw(p, oracle.bwd_input(p, chw_to(layout, dy), w))[0]
    expect = np.zeros((C, H, W))
    for kh in range(kH):
        for kw in range(kW):
            expect[:, ho + kh * d - pt, wo + kw * d - pl] += w[:, kh, kw]
    np.testing.assert_array_equal(dx, expect)


def test_one_by_one_kernel(oracle_mod):
    rng = np.random.default_rng(101)
    for layout in ("nhwc", "nchw"):
        shape = (2, 5, 7, 3) if layout == "nhwc" else (2, 3, 5, 7)
        x = rng.standard_normal(shape)
        w = rng.standard_normal((3, 1, 1))
        b = rng.standard_normal(3)
        p = oracle.problem(shape, 1, 1, 1, 1, 0, layout)
        y = to_nchw(p, oracle.fwd(p, x, w, b))
        ref = to_nchw(p, x) * w[None, :, :, :] + b[None, :, None, None]
        np.testing.assert_allclose(y, ref, rtol=1e-15)
        p2 = oracle.problem(shape, 1, 1, 2, 1, 0, layout)
        y2 = to_nchw(p2, oracle.fwd(p2, x, w, b))
        np.testing.assert_allclose(y2, ref[:, :, 0::2, 0::2], rtol=1e-15)


def test_separable_kernel(oracle_mod):
    """W[c] = u[c] (x) v[c]: the 2-D conv equals a kH x 1 conv of a 1 x kW conv
    (zero padding commutes with the separable sum), strides included."""
    rng = np.random.default_rng(111)
    for layout in ("nhwc", "nchw"):
        for (kH, kW, s, d, pads) in [(3, 5, 1, 1, (1, 1, 2, 2)), (4, 3, 2, 1, (2, 1, 0, 1)),
                                     (3, 3, (2, 3), 2, (0, 2, 1, 1))]:
            C = 3
            shape = (2, 9, 11, C) if layout == "nhwc" else (2, C, 9, 11)
            x = rng.standard_normal(shape)
            u = rng.standard_normal((C, kH))
            v = rng.standard_normal((C, kW))
            sh, sw = (s, s) if np.isscalar(s) else s
            pt, pb, pl, pr = pads
            p = oracle.problem(shape, kH, kW, (sh, sw), d, pads, layout)
            y = oracle.fwd(p, x, u[:, :, None] * v[:, None, :])
            pw = oracle.problem(shape, 1, kW, (1, sw), d, (0, 0, pl, pr), layout)
            t = oracle.fwd(pw, x, v[:, None, :])
            ph = oracle.problem(t.shape, kH, 1, (sh, 1), d, (pt, pb, 0, 0), layout)
            y2 = oracle.fwd(ph, t, u[:, :, None])
            np.testing.assert_allclose(y, y2, rtol=1e-12, atol=1e-12)


def test_sampled_evaluators_match_full(oracle_mod):
    for p, layout, rng in valid_cases(121, 30, max_hw=10, max_k=5):
        x = rng.standard_normal(oracle.in_shape(p))
        w = rng.standard_normal((int(p[3]), int(p[4]), int(p[5])))
        b = rng.standard_normal(int(p[3]))
        dy = rng.standard_normal(oracle.out_shape(p))
        y = oracle.fwd(p, x, w, b)
        dx = oracle.bwd_input(p, dy, w)
        iy = rng.integers(0, y.size, size=min(50, y.size))
        ix = rng.integers(0, dx.size, size=min(50, dx.size))
        np.testing.assert_allclose(oracle.fwd_at(p, x, w, b, iy), y.reshape(-1)[iy],
                                   rtol=1e-14, atol=1e-14)
        np.testing.assert_allclose(oracle.bwd_input_at(p, dy, w, ix), dx.reshape(-1)[ix],
                                   rtol=1e-12, atol=1e-12)


def test_bias_absent_is_zero(oracle_mod):
    rng = np.random.default_rng(131)
    p = oracle.problem((1, 5, 5, 3), 3, 3, 1, 1, "same", "nhwc")
    x = rng.standard_normal((1, 5, 5, 3))
    w = rng.standard_normal((3, 3, 3))
    np.testing.assert_array_equal(oracle.fwd(p, x, w, None), oracle.fwd(p, x, w, np.zeros(3)))


# ------------------------------------------------ weight / bias gradients --

def test_golden_weight_gradient(oracle_mod):
    g = load_golden("orientation_2x2.json")
    p = prob1(g["H"], g["W"], 1, g["kH"], g["kW"], g["stride"], g["dilation"], g["pads"])
    dw, db = oracle.bwd_weight(p, chw_to("nhwc", [g["x"]]), chw_to("nhwc", [g["bwd_weight"]["dy"]]))
    assert np.array_equal(dw[0], np.array(g["bwd_weight"]["dw"]))
    assert db[0] == g["bwd_weight"]["db"]
    g = load_golden("stride2_4x4.json")
    for layout in ("nhwc", "nchw"):
        for key in ("even", "xla_same"):
            case = g[key]
            p = prob1(4, 4, 1, 3, 3, case["stride"], 1, case["pads"], layout=layout)
            dw, db = oracle.bwd_weight(p, chw_to(layout, [g["x"]]), chw_to(layout, [case["dy"]]))
            assert np.array_equal(dw[0], np.array(case["dw"])), (layout, key)
            assert db[0] == case["db"]


def test_weight_gradient_equals_torch_autograd(oracle_mod):
    for p, layout, rng in valid_cases(141, 50):
        N, H, W, C, kH, kW, sh, sw, dh, dw_, pt, pb, pl, pr, _, _ = (int(v) for v in p)
        x = rng.standard_normal(oracle.in_shape(p))
        dy = rng.standard_normal(oracle.out_shape(p))
        wt = torch.from_numpy(rng.standard_normal((C, 1, kH, kW))).requires_grad_(True)
        bt = torch.from_numpy(rng.standard_normal(C)).requires_grad_(True)
        xn = torch.from_numpy(np.ascontiguousarray(to_nchw(p, x)))
        y = F.conv2d(F.pad(xn, (pl, pr, pt, pb)), wt, bt, (sh, sw), 0, (dh, dw_), groups=C)
        gw, gb = torch.autograd.grad(y, (wt, bt), torch.from_numpy(np.ascontiguousarray(to_nchw(p, dy))))
        dw, db = oracle.bwd_weight(p, x, dy)
        np.testing.assert_allclose(dw, gw.numpy()[:, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(db, gb.numpy(), rtol=1e-12, atol=1e-12)


def test_weight_gradient_linearity_identity(oracle_mod):
    """The forward is linear in (W, b) for fixed x, so
    <dW, V> + <db, u> = <dy, fwd(x; V, u)> for any V, u."""
    for p, layout, rng in valid_cases(151, 60, max_hw=12, max_k=5, max_c=4):
        C, kH, kW = int(p[3]), int(p[4]), int(p[5])
        x = rng.standard_normal(oracle.in_shape(p))
        dy = rng.standard_normal(oracle.out_shape(p))
        V = rng.standard_normal((C, kH, kW))
        u = rng.standard_normal(C)
        dw, db = oracle.bwd_weight(p, x, dy)
        lhs = float(np.sum(dw * V) + np.sum(db * u))
        rhs = float(np.sum(dy * oracle.fwd(p, x, V, u)))
        assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(rhs)), (lhs, rhs)


def test_bias_gradient_closed_form(oracle_mod):
    """db[c] = sum over n, h, w of dy[c] (the page's closed form)."""
    for p, layout, rng in valid_cases(161, 30):
        dy = rng.standard_normal(oracle.out_shape(p))
        _, db = oracle.bwd_weight(p, rng.standard_normal(oracle.in_shape(p)), dy)
        axes = (0, 1, 2) if layout == "nhwc" else (0, 2, 3)
        np.testing.assert_allclose(db, dy.sum(axis=axes), rtol=1e-13, atol=1e-13)


# ------------------------------------------- fused batch norm + activation ---

ACTS = ["none", "relu", "relu6", "silu"]


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_golden_bn_act(oracle_mod, layout):
    g = load_golden("bn_act_2ch.json")
    p = prob1(g["H"], g["W"], g["C"], g["kH"], g["kW"], 1, 1, g["pads"], layout=layout)
    x = chw_to(layout, g["x"])
    bn = (g["gamma"], g["beta"], g["mean"], g["var"], g["eps"])
    for act in ACTS:
        y = to_chw(layout, oracle.fwd_bn_act(p, x, g["w"], g["b"], bn, act))
        want = np.array(g["out"][act])
        tol = g["silu_tolerance"] if act == "silu" else 0.0
        assert np.allclose(y, want, rtol=0, atol=tol), (act, y, want)


def random_bn(rng, C):
    return (rng.uniform(-1.5, 1.5, C), rng.uniform(-0.5, 0.5, C), rng.uniform(-0.3, 0.3, C),
            rng.uniform(0.2, 2.0, C), float(rng.choice([1e-5, 1e-3, 0.1])))


def torch_bn_act(z_nchw, bn, act):
    g, be, mu, var = (torch.tensor(np.asarray(v), dtype=torch.float64) for v in bn[:4])
    eps = bn[4]
    u = F.batch_norm(torch.from_numpy(z_nchw), mu, var, g, be, training=False, eps=eps)
    return {"none": lambda t: t, "relu": F.relu, "relu6": F.relu6, "silu": F.silu}[act](u).numpy()


def test_bn_act_equals_torch_batch_norm_and_activations(oracle_mod):
    # the library's eval-mode batch norm and activation functions, float64
    rng = np.random.default_rng(404)
    for p, _, _ in valid_cases(405, 20):
        x = rng.uniform(-2, 2, oracle.in_shape(p))
        C = int(p[3])
        w = rng.normal(0, 1, (C, int(p[4]), int(p[5])))
        b = rng.uniform(-0.5, 0.5, C)
        bn = random_bn(rng, C)
        z = to_nchw(p, oracle.fwd(p, x, w, b))
        for act in ACTS:
            got = to_nchw(p, oracle.fwd_bn_act(p, x, w, b, bn, act))
            want = torch_bn_act(z, bn, act)
            assert np.allclose(got, want, rtol=1e-13, atol=1e-14), act


def test_bn_identity_statistics_reduce_to_plain_forward(oracle_mod):
    # gamma = sqrt(var + eps), beta = mean: the normalisation is the identity
    rng = np.random.default_rng(406)
    for p, _, _ in valid_cases(407, 10):
        C = int(p[3])
        x = rng.uniform(-1, 1, oracle.in_shape(p))
        w = rng.normal(0, 1, (C, int(p[4]), int(p[5])))
        var, eps = rng.uniform(0.5, 3, C), 1e-3
        mean = rng.uniform(-1, 1, C)
        bn = (np.sqrt(var + eps), mean, mean, var, eps)
        y = oracle.fwd(p, x, w, None)
        assert np.allclose(oracle.fwd_bn_act(p, x, w, None, bn, "none"), y, rtol=1e-13, atol=1e-13)
        assert np.array_equal(oracle.fwd_bn_act(p, x, w, None, None, "relu"), np.maximum(y, 0))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_bn_act_constant_input_closed_form(oracle_mod, layout):
    # x = a everywhere, 3x3 SAME: an interior output is a*sum(W[c]) + b[c]
    a, C = 0.75, 3
    p = oracle.problem((1, 5, 5, C) if layout == "nhwc" else (1, C, 5, 5), 3, 3, layout=layout)
    w = np.arange(C * 9, dtype=np.float64).reshape(C, 3, 3) / 20.0 - 0.4
    b = np.array([0.1, -0.2, 0.3])
    bn = ([1.5, -2.0, 0.5], [0.25, 0.0, -1.0], [1.0, -0.5, 2.0], [0.44, 3.0, 0.01], 0.06)
    for act in ACTS:
        y = to_chw(layout, oracle.fwd_bn_act(p, np.full(oracle.in_shape(p), a), w, b, bn, act))
        for c in range(C):
            z = a * w[c].sum() + b[c]
            u = bn[0][c] * (z - bn[2][c]) / np.sqrt(bn[3][c] + bn[4]) + bn[1][c]
            want = {"none": u, "relu": max(u, 0.0), "relu6": min(max(u, 0.0), 6.0),
                    "silu": u / (1.0 + np.exp(-u))}[act]
            assert abs(y[c, 2, 2] - want) <= 1e-12 * max(1.0, abs(want)), (act, c)


# ---------------------------------------------------- channel multiplier ---

def mult_cases(seed, count, **kw):
    """Random valid problems with a channel multiplier M in 2..4."""
    out = []
    for p, layout, rng in valid_cases(seed, count, **kw):
        p = p.copy()
        p[15] = int(rng.integers(2, 5))
        out.append((p, layout, rng))
    return out


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_golden_multiplier(oracle_mod, layout):
    g = load_golden("multiplier_2x.json")
    shape = (1, g["H"], g["W"], g["C"]) if layout == "nhwc" else (1, g["C"], g["H"], g["W"])
    p = oracle.problem(shape, g["kH"], g["kW"], 1, 1, tuple(g["pads"]), layout,
                       multiplier=g["M"])
    x = chw_to(layout, [g["x"]])
    y = oracle.fwd(p, x, g["w"], g["b"])
    assert np.array_equal(to_chw(layout, y), np.array(g["y"]))
    dx = oracle.bwd_input(p, chw_to(layout, g["bwd"]["dy"]), g["w"])
    assert np.array_equal(to_chw(layout, dx)[0], np.array(g["bwd"]["dx"]))
    idx = np.arange(dx.size)
    assert np.array_equal(oracle.bwd_input_at(p, chw_to(layout, g["bwd"]["dy"]), g["w"], idx),
                          dx.reshape(-1))
    dw, db = oracle.bwd_weight(p, x, chw_to(layout, g["wgrad"]["dy"]))
    assert np.array_equal(dw, np.array(g["wgrad"]["dw"]))
    assert np.array_equal(db, np.array(g["wgrad"]["db"]))


@pytest.mark.parametrize("dense", [False, True])
def test_multiplier_equals_torch_grouped_conv(oracle_mod, dense):
    # the library's grouped conv (groups = C, C*M output channels), float64
    for p, layout, rng in mult_cases(171, 30):
        Co = oracle.out_channels(p)
        x = rng.standard_normal(oracle.in_shape(p))
        w = rng.standard_normal((Co, int(p[4]), int(p[5])))
        b = rng.standard_normal(Co)
        np.testing.assert_allclose(oracle.fwd(p, x, w, b), torch_fwd(p, x, w, b, dense),
                                   rtol=1e-12, atol=1e-12)


def test_multiplier_gradients_equal_torch_autograd(oracle_mod):
    for p, layout, rng in mult_cases(181, 30):
        N, H, W, C, kH, kW, sh, sw, dh, dw_, pt, pb, pl, pr, _, M = (int(v) for v in p)
        x = rng.standard_normal(oracle.in_shape(p))
        dy = rng.standard_normal(oracle.out_shape(p))
        xt = torch.from_numpy(np.ascontiguousarray(to_nchw(p, x))).requires_grad_(True)
        wt = torch.from_numpy(rng.standard_normal((C * M, 1, kH, kW))).requires_grad_(True)
        bt = torch.from_numpy(rng.standard_normal(C * M)).requires_grad_(True)
        y = F.conv2d(F.pad(xt, (pl, pr, pt, pb)), wt, bt, (sh, sw), 0, (dh, dw_), groups=C)
        gx, gw, gb = torch.autograd.grad(y, (xt, wt, bt),
                                         torch.from_numpy(np.ascontiguousarray(to_nchw(p, dy))))
        w = wt.detach().numpy()[:, 0]
        np.testing.assert_allclose(to_nchw(p, oracle.bwd_input(p, dy, w)), gx.numpy(),
                                   rtol=1e-12, atol=1e-12)
        dw, db = oracle.bwd_weight(p, x, dy)
        np.testing.assert_allclose(dw, gw.numpy()[:, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(db, gb.numpy(), rtol=1e-12, atol=1e-12)


def test_multiplier_is_depthwise_of_repeated_channels(oracle_mod):
    """With M output channels per input channel, the forward equals the plain
    depthwise forward of x with every channel repeated M times, and the input
    gradient is that forward's input gradient summed over each channel's M
    copies."""
    for p, layout, rng in mult_cases(191, 30):
        M = int(p[15])
        x = rng.standard_normal(oracle.in_shape(p))
        Co = oracle.out_channels(p)
        w = rng.standard_normal((Co, int(p[4]), int(p[5])))
        b = rng.standard_normal(Co)
        dy = rng.standard_normal(oracle.out_shape(p))
        axis = 3 if layout == "nhwc" else 1
        x_rep = np.repeat(x, M, axis=axis)
        p1 = oracle.problem(x_rep.shape, int(p[4]), int(p[5]), (int(p[6]), int(p[7])),
                            (int(p[8]), int(p[9])), tuple(int(v) for v in p[10:14]), layout)
        assert np.array_equal(oracle.fwd(p, x, w, b), oracle.fwd(p1, x_rep, w, b))
        dx1 = oracle.bwd_input(p1, dy, w)
        shape = list(dx1.shape)
        shape[axis:axis + 1] = [shape[axis] // M, M]
        np.testing.assert_allclose(oracle.bwd_input(p, dy, w),
                                   dx1.reshape(shape).sum(axis=axis + 1), rtol=1e-13, atol=1e-13)
        dw, db = oracle.bwd_weight(p, x, dy)
        dw1, db1 = oracle.bwd_weight(p1, x_rep, dy)
        np.testing.assert_allclose(dw, dw1, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(db, db1, rtol=1e-13, atol=1e-13)


def test_multiplier_adjoint_identity(oracle_mod):
    for p, layout, rng in mult_cases(201, 40, max_hw=10, max_k=4, max_c=3):
        x = rng.standard_normal(oracle.in_shape(p))
        w = rng.standard_normal((oracle.out_channels(p), int(p[4]), int(p[5])))
        dy = rng.standard_normal(oracle.out_shape(p))
        lhs = float(np.sum(dy * oracle.fwd(p, x, w)))
        rhs = float(np.sum(oracle.bwd_input(p, dy, w) * x))
        assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), (lhs, rhs)
        idx = rng.integers(0, x.size, size=50)
        np.testing.assert_allclose(oracle.bwd_input_at(p, dy, w, idx),
                                   oracle.bwd_input(p, dy, w).reshape(-1)[idx],
                                   rtol=1e-12, atol=1e-12)
        oidx = rng.integers(0, dy.size, size=50)
        np.testing.assert_allclose(oracle.fwd_at(p, x, w, None, oidx),
                                   oracle.fwd(p, x, w).reshape(-1)[oidx], rtol=1e-12, atol=1e-12)
