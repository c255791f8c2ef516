"""GPU parity of the forward with the fused batch-norm / activation epilogue.

Reference: the float64 oracle's forward followed by its inference-mode batch
norm and activation.  Error rule, from the arithmetic of the fused path (per
channel s = gamma / sqrt(var + eps) and t = beta - mean * s in f32; the tiled
kernels fold them into the filter and bias, W' = s * W and b' = s * b + t,
the direct kernel applies fmaf(z, s, t) to z = forward + bias; then the
activation):
    |gpu - ref| <= L * 1e-5 * S + 8 * 2**-24 * |ref|
with S = |s| * (sum|x*W| + |b| + |mean|) + |beta|, s = gamma / sqrt(var + eps),
L = 1.1 for silu (its Lipschitz bound) and 1 otherwise; the last term covers
silu's own rounding: expf (2 ulp), the add, and the fast division (2 ulp).  Where S = 0 the values must be
equal.  Bit-level checks: with the identity statistics absent and relu /
relu6, the fused kernel returns exactly relu(fwd) / relu6(fwd) of the plain
kernel (scale 1 and shift -0 leave filter, bias and z untouched), and f16 weights
give the same bits as their f32 copies.
"""
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

ACTS = ["none", "relu", "relu6", "silu"]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dwbuild.build()
    dw.lib()
    yield
    torch.cuda.synchronize()
    assert dw.dwconv2d_take_device_error() == 0


def bn_of(case):
    return wl.make_bn(case.Co, case.seed + 500)


def bound(case, inp, bn, act, idx=None):
    """(ref, allowed error) at all outputs (idx None) or at flat indices idx."""
    p = gu.problem(case)
    x, w, b = gu.f64(inp["x"]), gu.f64(inp["w32"]), gu.f64(inp["b"])
    bn64 = None if bn is None else tuple(gu.f64(t) for t in bn[:4]) + (bn[4],)
    if idx is None:
        z = oracle.fwd(p, x, w, b)
        terms = oracle.fwd(p, np.abs(x), np.abs(w), None if b is None else np.abs(b))
        ch = oracle.channel_of(p, np.arange(z.size))
    else:
        z = oracle.fwd_at(p, x, w, b, idx)
        terms = oracle.fwd_at(p, np.abs(x), np.abs(w), None if b is None else np.abs(b), idx)
        ch = oracle.channel_of(p, idx)
    ref = oracle.bn_act(p, z, idx, bn64, act)
    if bn64 is None:
        S = terms.reshape(-1)
    else:
        g, be, mu, var, eps = bn64
        s = np.abs(g / np.sqrt(var + eps))
        S = s[ch] * (terms.reshape(-1) + np.abs(mu)[ch]) + np.abs(be)[ch]
    L = 1.1 if act == "silu" else 1.0
    tol = L * gu.TOL * S + 8 * 2.0 ** -24 * np.abs(ref.reshape(-1))
    return ref.reshape(-1), tol


def gpu_fused(case, inp, bn, act, algo="auto", w_key="w"):
    x = inp["x"].cuda()
    w = inp[w_key].cuda()
    b = None if inp["b"] is None else inp["b"].cuda()
    bnd = None if bn is None else tuple(t.cuda() for t in bn[:4]) + (bn[4],)
    return dw.dwconv2d_fwd_bn_act(x, w, b, bnd, act, stride=case.stride, dilation=case.dilation,
                                  padding=case.padding, layout=case.layout, algo=algo)


def check_close(got, ref, tol, what):
    g = got.detach().cpu().numpy().astype(np.float64).reshape(-1)
    assert g.shape == ref.shape, what
    assert np.all(np.isfinite(g)), what
    err = np.abs(g - ref)
    zero = tol == 0
    assert np.array_equal(g[zero], ref[zero]), f"{what}: term-free outputs differ"
    bad = err > tol
    if bad.any():
        i = int(np.flatnonzero(bad)[0])
        raise AssertionError(f"{what}: |gpu-ref| {err[i]:.3e} > {tol[i]:.3e} at {i} "
                             f"(gpu {g[i]!r}, ref {ref[i]!r}), {int(bad.sum())} elements")


def check(case, acts=ACTS, algos=("auto", "direct"), with_bn=(True, False)):
    inp = gu.inputs(case)
    for use_bn in with_bn:
        bn = bn_of(case) if use_bn else None
        for act in acts:
            if bn is None and act == "none":
                continue
            ref, tol = bound(case, inp, bn, act)
            for algo in algos:
                y = gpu_fused(case, inp, bn, act, algo)
                torch.cuda.synchronize()
                check_close(y, ref, tol, f"{case.name} bn={use_bn} act={act} [{algo}]")


CONFIGS = wl.tiny() + wl.mobilenet() + [c for c in wl.conformer() if c.W == 24] + \
    [c for c in wl.large() if c.H == 30]


@pytest.mark.parametrize("case", CONFIGS, ids=lambda c: c.name)
def test_config_cases(case):
    check(case)


# one case per tiled forward kernel instance (both layouts), ragged edges
TILED = [
    Case("e_3x3", 2, 37, 45, 72, 3, 3, seed=91),
    Case("e_3x3_big", 4, 64, 64, 128, 3, 3, seed=92),
    Case("e_3x3_s2", 4, 29, 41, 44, 3, 3, stride=2, padding=1, seed=93),
    Case("e_3x3_d2", 2, 23, 30, 36, 3, 3, dilation=2, seed=94),
    Case("e_5x5", 2, 17, 39, 68, 5, 5, seed=95),
    Case("e_7x7", 2, 19, 23, 36, 7, 7, seed=96),
    Case("e_1x15", 4, 2, 300, 44, 1, 15, act="normal", seed=97),
    Case("e_1x31", 3, 3, 290, 68, 1, 31, act="normal", seed=98),
    Case("e_nchw_3x3", 2, 37, 44, 20, 3, 3, layout="nchw", seed=99),
    Case("e_nchw_5x5", 2, 35, 52, 10, 5, 5, layout="nchw", seed=100),
    Case("e_nchw_7x7", 2, 33, 28, 9, 7, 7, layout="nchw", seed=101),
    Case("e_nchw_1x31", 2, 1, 300, 40, 1, 31, act="normal", layout="nchw", seed=102),
    Case("e_nchw_1x31_ragged", 2, 1, 292, 40, 1, 31, padding=(0, 0, 15, 14), act="normal",
         layout="nchw", seed=103),
]


@pytest.mark.parametrize("case", TILED, ids=lambda c: c.name)
def test_tiled_kernels(case):
    inp = gu.inputs(case)
    x = inp["x"].cuda()
    y = torch.empty(case.out_shape(*gu.out_hw(case)), device="cuda")
    assert gu.chosen_algo(case, 0, x, inp["w"].cuda(), y) == dw.DW_ALGO_TILED
    check(case, algos=("tiled",))


@pytest.mark.parametrize("case", [TILED[0], TILED[2], TILED[7], TILED[8], TILED[11]],
                         ids=lambda c: c.name)
def test_plain_activation_is_bit_exact(case):
    inp = gu.inputs(case)
    plain = gu.gpu_fwd(case, inp)
    relu = gpu_fused(case, inp, None, "relu")
    relu6 = gpu_fused(case, inp, None, "relu6")
    torch.cuda.synchronize()
    assert torch.equal(relu, torch.where(plain < 0, torch.zeros_like(plain), plain))
    assert torch.equal(relu6, torch.clamp(plain, 0.0, 6.0))


@pytest.mark.parametrize("case", [TILED[1], TILED[6], TILED[9]], ids=lambda c: c.name)
def test_f16_weights_bit_identical(case):
    c16 = case.with_(wtype="f16")
    inp = gu.inputs(c16)
    bn = bn_of(c16)
    for act in ACTS:
        a = gpu_fused(c16, inp, bn, act, w_key="w")
        b = gpu_fused(c16, inp, bn, act, w_key="w32")
        torch.cuda.synchronize()
        assert torch.equal(a, b), act


def test_full_size_sampled():
    rng = np.random.default_rng(17)
    cases = [c for c in wl.large() if c.H == 512] + [wl.mobilenet()[2]] + \
        [c for c in wl.conformer() if c.W == 512]
    for case in cases:
        inp = gu.inputs(case)
        bn = bn_of(case)
        act = "relu6" if case.kH == 3 else "silu"
        y = gpu_fused(case, inp, bn, act)
        torch.cuda.synchronize()
        idx = gu.structured_sample(tuple(y.shape), case.layout, rng, count=4000)
        ref, tol = bound(case, inp, bn, act, idx)
        got = y.reshape(-1)[torch.from_numpy(idx).cuda()]
        check_close(got, ref, tol, f"{case.name} sampled")
