"""Helpers for the GPU parity tests: oracle references with their error
scales and the comparison rule.

Comparison rule (float32 kernels against the float64 oracle): per element
    |gpu - ref| <= 1e-5 * scale
where scale is the sum of the magnitudes of the terms that make the element:
sum over taps |x * W| + |b| for the forward, sum |W * dy| for the input
gradient.  The oracle computes the scale exactly by running on |x|, |W|,
|b| (every term is then non-negative, so the sum of magnitudes is the output
itself).  Where the scale is 0 (no term at all, e.g. an output that sees only
padding and no bias) the GPU value must equal the reference exactly.
"""
import numpy as np
import torch

import oracle
import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200.workloads import Case, make_inputs

TOL = 1e-5


def problem(case: Case):
    return oracle.problem(case.in_shape(), case.kH, case.kW, case.stride, case.dilation,
                          case.padding, case.layout, multiplier=case.multiplier)


def out_hw(case: Case):
    o = oracle.out_shape(problem(case))
    return (o[1], o[2]) if case.layout == "nhwc" else (o[2], o[3])


def inputs(case: Case):
    return make_inputs(case, out_hw(case))


def f64(t):
    return None if t is None else t.detach().cpu().numpy().astype(np.float64)


def reference_fwd(case, inp):
    p = problem(case)
    x, w, b = f64(inp["x"]), f64(inp["w32"]), f64(inp["b"])
    ref = oracle.fwd(p, x, w, b)
    scale = oracle.fwd(p, np.abs(x), np.abs(w), None if b is None else np.abs(b))
    return ref, scale


def reference_bwd(case, inp):
    p = problem(case)
    dy, w = f64(inp["dy"]), f64(inp["w32"])
    return oracle.bwd_input(p, dy, w), oracle.bwd_input(p, np.abs(dy), np.abs(w))


def reference_fwd_at(case, inp, idx):
    p = problem(case)
    x, w, b = f64(inp["x"]), f64(inp["w32"]), f64(inp["b"])
    return (oracle.fwd_at(p, x, w, b, idx),
            oracle.fwd_at(p, np.abs(x), np.abs(w), None if b is None else np.abs(b), idx))


def reference_bwd_at(case, inp, idx):
    p = problem(case)
    dy, w = f64(inp["dy"]), f64(inp["w32"])
    return oracle.bwd_input_at(p, dy, w, idx), oracle.bwd_input_at(p, np.abs(dy), np.abs(w), idx)


def assert_close(gpu, ref, scale, what=""):
    g = np.asarray(gpu, dtype=np.float64).reshape(-1)
    r = np.asarray(ref, dtype=np.float64).reshape(-1)
    s = np.asarray(scale, dtype=np.float64).reshape(-1)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    zero = s == 0
    if zero.any():
        assert np.array_equal(g[zero], r[zero]), f"{what}: terms-free outputs differ"
    nz = ~zero
    ratio = np.abs(g[nz] - r[nz]) / s[nz]
    if ratio.size:
        worst = int(np.argmax(ratio))
        assert ratio[worst] <= TOL, (
            f"{what}: max |gpu-ref|/sum|terms| = {ratio[worst]:.3e} > {TOL} at flat "
            f"{np.flatnonzero(nz)[worst]} (gpu {g[nz][worst]!r}, ref {r[nz][worst]!r})")


def gpu_fwd(case, inp, algo="auto", w_key="w", out=None, device="cuda"):
    x = inp["x"].to(device)
    w = inp[w_key].to(device)
    b = None if inp["b"] is None else inp["b"].to(device)
    return dw.dwconv2d_fwd(x, w, b, stride=case.stride, dilation=case.dilation,
                           padding=case.padding, layout=case.layout, algo=algo, out=out)


def gpu_bwd(case, inp, algo="auto", w_key="w", out=None, device="cuda"):
    dy = inp["dy"].to(device)
    w = inp[w_key].to(device)
    return dw.dwconv2d_bwd_input(dy, w, (case.H, case.W), stride=case.stride,
                                 dilation=case.dilation, padding=case.padding,
                                 layout=case.layout, algo=algo, out=out,
                                 multiplier=case.multiplier)


def desc_of(case, algo="auto"):
    return dw.make_desc(case.N, case.H, case.W, case.C, case.kH, case.kW, stride=case.stride,
                        dilation=case.dilation, padding=case.padding, layout=case.layout,
                        wtype=case.wtype, algo=algo, multiplier=case.multiplier)


def chosen_algo(case, op, t_in, t_w, t_out, algo="auto"):
    return dw.dwconv2d_query_algo(desc_of(case, algo), op, t_in.data_ptr(), t_w.data_ptr(),
                                  t_out.data_ptr())


def structured_sample(shape, layout, rng, count=20000):
    """Flat indices of a 4-D tensor: random positions plus every border row
    and column of a few (n, c) slices, the places padding and tile edges meet."""
    if layout == "nhwc":
        N, H, W, C = shape
    else:
        N, C, H, W = shape
    idx = [rng.integers(0, N * H * W * C, size=count)]
    for _ in range(4):
        n, c = int(rng.integers(0, N)), int(rng.integers(0, C))
        hs = np.array(sorted({0, 1, H // 2, H - 2, H - 1} & set(range(H))))
        ws = np.arange(W)
        for h_list, w_list in ((hs, ws), (np.arange(H), np.array(sorted({0, 1, W - 2, W - 1} & set(range(W)))))):
            hh, ww = np.meshgrid(h_list, w_list, indexing="ij")
            hh, ww = hh.reshape(-1), ww.reshape(-1)
            if layout == "nhwc":
                flat = ((n * H + hh) * W + ww) * C + c
            else:
                flat = ((n * C + c) * H + hh) * W + ww
            idx.append(flat)
    return np.unique(np.concatenate(idx).astype(np.int64))
