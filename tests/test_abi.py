"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, resolves pads and output extents exactly as the oracle's
(separately written) rules do, and rejects invalid or aliasing calls before
touching CUDA.  No call here reaches a kernel launch."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import depthwise_convolution_fwd_b200 as dw
from depthwise_convolution_fwd_b200 import build as dwbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dwbuild.build()
    return dw.lib()


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"\b(dwconv2d_\w+)\s*\(", text))
    return sorted(names)


def test_exports_every_declared_symbol(lib):
    declared = header_functions()
    assert "dwconv2d_fwd" in declared and "dwconv2d_bwd_input" in declared
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert sorted(dw.EXPORTS) == declared


def test_version_and_status_strings(lib):
    assert dw.dwconv2d_version() >= 10000
    for st in range(7):
        assert dw.status_string(st).startswith("DW_")


def random_desc(rng):
    N, H, W, C = (int(v) for v in rng.integers(1, 40, size=4))
    kH, kW = (int(v) for v in rng.integers(1, 8, size=2))
    s = tuple(int(v) for v in rng.integers(1, 4, size=2))
    d = tuple(int(v) for v in rng.integers(1, 4, size=2))
    pad = "same" if rng.random() < 0.5 else tuple(int(v) for v in rng.integers(0, 5, size=4))
    layout = "nhwc" if rng.random() < 0.5 else "nchw"
    return (N, H, W, C, kH, kW, s, d, pad, layout)


def test_out_shape_and_pads_match_oracle(lib):
    rng = np.random.default_rng(7)
    checked = 0
    for _ in range(3000):
        N, H, W, C, kH, kW, s, d, pad, layout = random_desc(rng)
        shape = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
        p = oracle.problem(shape, kH, kW, s, d, pad, layout)
        desc = dw.make_desc(N, H, W, C, kH, kW, stride=s, dilation=d, padding=pad, layout=layout)
        o = oracle.out_shape(p)
        Ho, Wo = (o[1], o[2]) if layout == "nhwc" else (o[2], o[3])
        if Ho < 1 or Wo < 1:
            with pytest.raises(dw.DwError) as e:
                dw.dwconv2d_out_shape(desc)
            assert e.value.status == dw.DW_ERR_INVALID_ARG
            continue
        assert dw.dwconv2d_out_shape(desc) == (Ho, Wo)
        assert dw.dwconv2d_resolved_pads(desc) == tuple(int(v) for v in p[10:14])
        checked += 1
    assert checked > 1500


BAD = [
    dict(N=0), dict(H=0), dict(W=-1), dict(C=0), dict(kH=0), dict(kW=-2),
    dict(stride_h=0), dict(stride_w=-1), dict(dil_h=0), dict(dil_w=0),
    dict(pad_mode=2), dict(pad_mode=0, pad_top=-1), dict(pad_mode=0, pad_right=-3),
    dict(layout=2), dict(wtype=5), dict(wtype=2), dict(atype=3), dict(atype=-1),
    dict(algo=3), dict(algo=-1),
    dict(kH=9, pad_mode=0),  # no output row left: Ho = 0
]


@pytest.mark.parametrize("bad", BAD)
def test_invalid_descriptors_rejected_before_launch(lib, bad):
    desc = dw.make_desc(1, 8, 8, 4, 3, 3)
    for k, v in bad.items():
        setattr(desc, k, v)
    fake = 1 << 40  # never dereferenced: validation fails first
    assert dw.fwd_raw(desc, fake, fake + (1 << 20), None, fake + (2 << 20), 0) == dw.DW_ERR_INVALID_ARG
    assert dw.bwd_input_raw(desc, fake, fake + (1 << 20), fake + (2 << 20), 0) == dw.DW_ERR_INVALID_ARG
    assert dw.dwconv2d_query_algo(desc, 0, fake, fake + (1 << 20), fake + (2 << 20)) == -dw.DW_ERR_INVALID_ARG


def test_null_pointers_rejected(lib):
    desc = dw.make_desc(1, 8, 8, 4, 3, 3)
    fake = 1 << 40
    assert dw.fwd_raw(desc, 0, fake, None, fake + 4096, 0) == dw.DW_ERR_INVALID_ARG
    assert dw.fwd_raw(desc, fake, 0, None, fake + 4096, 0) == dw.DW_ERR_INVALID_ARG
    assert dw.fwd_raw(desc, fake, fake + 4096, None, 0, 0) == dw.DW_ERR_INVALID_ARG
    assert lib.dwconv2d_fwd(None, fake, fake, None, fake, None) == dw.DW_ERR_INVALID_ARG


def test_aliasing_rejected_before_launch(lib):
    # 1x8x8x4 NHWC, 3x3 SAME: x and y are 1 KiB each
    desc = dw.make_desc(1, 8, 8, 4, 3, 3)
    base = 1 << 40
    w = base + (1 << 20)
    assert dw.fwd_raw(desc, base, w, None, base, 0) == dw.DW_ERR_ALIAS            # in place
    assert dw.fwd_raw(desc, base, w, None, base + 1020, 0) == dw.DW_ERR_ALIAS     # partial overlap
    assert dw.fwd_raw(desc, base + 1020, w, None, base, 0) == dw.DW_ERR_ALIAS
    assert dw.fwd_raw(desc, base, w, None, w - 100, 0) == dw.DW_ERR_ALIAS         # y over w
    assert dw.fwd_raw(desc, base, w, w + 4096, w + 4096 - 8, 0) == dw.DW_ERR_ALIAS  # y over b
    assert dw.bwd_input_raw(desc, base, w, base + 512, 0) == dw.DW_ERR_ALIAS
    # adjacent but disjoint buffers are fine (query does not launch)
    assert dw.dwconv2d_query_algo(desc, 0, base, w, base + 1024) > 0


def q(desc, op=0, align=0):
    base = (1 << 40) + align
    return dw.dwconv2d_query_algo(desc, op, base, base + (1 << 30), base + (2 << 30))


def test_query_algo_selects_tiled_for_covered_shapes(lib):
    T, D = dw.DW_ALGO_TILED, dw.DW_ALGO_DIRECT
    # NHWC, C % 4 == 0, aligned: tiled for the instantiated kernel shapes
    assert q(dw.make_desc(1, 512, 512, 256, 3, 3)) == T
    assert q(dw.make_desc(1, 512, 512, 256, 3, 3), op=1) == T
    assert q(dw.make_desc(32, 56, 56, 144, 3, 3, stride=2, padding=1)) == T
    assert q(dw.make_desc(32, 56, 56, 144, 3, 3, stride=2, padding=1), op=1) == T
    assert q(dw.make_desc(16, 1, 512, 512, 1, 31)) == T
    assert q(dw.make_desc(1, 56, 56, 128, 5, 5)) == T
    # NCHW stride 1 with W % 4 == 0
    assert q(dw.make_desc(1, 512, 512, 256, 3, 3, layout="nchw")) == T
    assert q(dw.make_desc(16, 1, 512, 512, 1, 31, layout="nchw"), op=1) == T
    # not covered -> direct
    assert q(dw.make_desc(1, 13, 17, 7, 3, 3)) == D                      # C % 4 != 0
    assert q(dw.make_desc(1, 30, 19, 128, 7, 7, layout="nchw")) == D     # W % 4 != 0
    assert q(dw.make_desc(1, 16, 16, 8, 3, 3), align=4) == D             # unaligned pointers
    assert q(dw.make_desc(1, 16, 16, 8, 2, 2)) == D                      # no 2x2 instance
    assert q(dw.make_desc(1, 16, 16, 8, 3, 3, layout="nchw", stride=2)) == T        # strided fwd
    assert q(dw.make_desc(1, 16, 16, 8, 3, 3, layout="nchw", stride=2), op=1) == T  # strided bwd
    assert q(dw.make_desc(1, 16, 12, 8, 3, 3, layout="nchw", stride=2), op=1) == D  # Wo = 6
    assert q(dw.make_desc(1, 16, 16, 8, 5, 5, layout="nchw", stride=2)) == D
    # forcing
    assert q(dw.make_desc(1, 13, 17, 7, 3, 3, algo="direct")) == D
    assert q(dw.make_desc(1, 512, 512, 256, 3, 3, algo="direct")) == D
    assert q(dw.make_desc(1, 13, 17, 7, 3, 3, algo="tiled")) == -dw.DW_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 8, 8, 4)
    w = torch.zeros(4, 3, 3)
    with pytest.raises(TypeError):
        dw.dwconv2d_fwd(x, w)


def test_weight_gradient_host_checks(lib):
    desc = dw.make_desc(2, 16, 16, 32, 3, 3)
    need = dw.dwconv2d_bwd_weight_workspace_size(desc)
    assert need > 0
    # the workspace size depends on the problem only
    assert need == dw.dwconv2d_bwd_weight_workspace_size(dw.make_desc(2, 16, 16, 32, 3, 3))
    base = 1 << 40
    x, dy, dwp, db, ws = base, base + (1 << 24), base + (2 << 24), base + (3 << 24), base + (4 << 24)
    # too small a workspace, NULL tensors, invalid descriptor: rejected before launch
    assert dw.bwd_weight_raw(desc, x, dy, dwp, db, ws, need - 1, 0) == dw.DW_ERR_INVALID_ARG
    assert dw.bwd_weight_raw(desc, 0, dy, dwp, db, ws, need, 0) == dw.DW_ERR_INVALID_ARG
    assert dw.bwd_weight_raw(desc, x, dy, dwp, db, 0, need, 0) == dw.DW_ERR_INVALID_ARG
    bad = dw.make_desc(2, 16, 16, 32, 3, 3)
    bad.C = 0
    assert dw.bwd_weight_raw(bad, x, dy, dwp, db, ws, need, 0) == dw.DW_ERR_INVALID_ARG
    # outputs overlapping inputs or each other
    assert dw.bwd_weight_raw(desc, x, dy, x + 64, db, ws, need, 0) == dw.DW_ERR_ALIAS
    assert dw.bwd_weight_raw(desc, x, dy, dwp, dy + 4, ws, need, 0) == dw.DW_ERR_ALIAS
    assert dw.bwd_weight_raw(desc, x, dy, dwp, db, dwp + 8, need, 0) == dw.DW_ERR_ALIAS
    assert dw.bwd_weight_raw(desc, x, dy, dwp, db, x, need, 0) == dw.DW_ERR_ALIAS
    # kernel family selection (op 2 = weight gradient; no launch)
    T, D = dw.DW_ALGO_TILED, dw.DW_ALGO_DIRECT
    assert dw.dwconv2d_query_algo(desc, 2, x, dy, dwp) == T
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 16, 32, 3, 3, layout="nchw"), 2, x, dy, dwp) == T
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 16, 32, 7, 7, layout="nchw"), 2, x, dy, dwp) == T
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 18, 32, 3, 3, layout="nchw"), 2, x, dy, dwp) == D
    assert dw.dwconv2d_query_algo(
        dw.make_desc(2, 16, 16, 32, 3, 3, stride=2, layout="nchw"), 2, x, dy, dwp) == T
    assert dw.dwconv2d_query_algo(
        dw.make_desc(2, 16, 16, 32, 5, 5, stride=2, layout="nchw"), 2, x, dy, dwp) == D
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 16, 32, 1, 31, layout="nchw"), 2, x, dy, dwp) == T
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 18, 32, 1, 31, layout="nchw"), 2, x, dy, dwp) == D
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 16, 32, 1, 9, layout="nchw"), 2, x, dy, dwp) == D
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 16, 7, 3, 3), 2, x, dy, dwp) == D
    assert dw.dwconv2d_query_algo(dw.make_desc(2, 16, 16, 32, 3, 3, dilation=2), 2, x, dy, dwp) == D


def test_fused_epilogue_host_checks(lib):
    desc = dw.make_desc(1, 8, 8, 4, 3, 3)  # y: 1 KiB
    base = 1 << 40
    x, w, y = base, base + (1 << 20), base + (2 << 20)
    st = [base + (3 << 20) + 4096 * i for i in range(4)]
    R = dw.fwd_bn_act_raw
    # mixed NULL statistics, bad eps, unknown activation: rejected before launch
    for k in range(4):
        part = list(st)
        part[k] = 0
        assert R(desc, x, w, None, part, 1e-5, dw.DW_ACT_RELU, y, 0) == dw.DW_ERR_INVALID_ARG
    for eps in (-1e-3, float("nan"), float("inf")):
        assert R(desc, x, w, None, st, eps, dw.DW_ACT_NONE, y, 0) == dw.DW_ERR_INVALID_ARG
    for act in (-1, 4):
        assert R(desc, x, w, None, st, 1e-5, act, y, 0) == dw.DW_ERR_INVALID_ARG
    # y over any statistics array, or over x / w / b
    for k in range(4):
        part = list(st)
        part[k] = y + 512
        assert R(desc, x, w, None, part, 1e-5, dw.DW_ACT_NONE, y, 0) == dw.DW_ERR_ALIAS
    assert R(desc, x, w, None, st, 1e-5, dw.DW_ACT_NONE, x + 8, 0) == dw.DW_ERR_ALIAS
    assert R(desc, x, w, y + 16, st, 1e-5, dw.DW_ACT_NONE, y, 0) == dw.DW_ERR_ALIAS
    # invalid descriptor
    bad = dw.make_desc(1, 8, 8, 4, 3, 3)
    bad.kH = 0
    assert R(bad, x, w, None, st, 1e-5, dw.DW_ACT_NONE, y, 0) == dw.DW_ERR_INVALID_ARG


def test_channel_multiplier_host_checks(lib):
    # 0 and 1 both mean the plain depthwise convolution; negative or huge: invalid
    fake = 1 << 40
    for m, ok in ((0, True), (1, True), (3, True), (-1, False), (5000, False)):
        d = dw.make_desc(1, 8, 8, 4, 3, 3, multiplier=m)
        if ok:
            assert dw.dwconv2d_out_shape(d) == (8, 8)
        else:
            with pytest.raises(dw.DwError):
                dw.dwconv2d_out_shape(d)
            assert dw.fwd_raw(d, fake, fake + (1 << 20), None, fake + (2 << 20), 0) == dw.DW_ERR_INVALID_ARG
    # sizes use C*M output channels: x 1 KiB, y 2 KiB (M = 2)
    d = dw.make_desc(1, 8, 8, 4, 3, 3, multiplier=2)
    base = 1 << 40
    w = base + (1 << 20)
    assert dw.dwconv2d_query_algo(d, 0, base, w, base + 1024) > 0          # adjacent: fine
    assert dw.fwd_raw(d, base, w, None, w - 2047, 0) == dw.DW_ERR_ALIAS      # y (2 KiB) over w
    assert dw.fwd_raw(d, base, w, w + 4096, w + 4096 - 2040, 0) == dw.DW_ERR_ALIAS  # y over b
    assert dw.bwd_input_raw(d, base, w, base + 2040, 0) == dw.DW_ERR_ALIAS   # dx over dy (2 KiB)
    # filter of C*M rows: a y placed right after a 4*9*4-byte filter would overlap an 8-row one
    assert dw.fwd_raw(d, base, w, None, w + 4 * 9 * 4, 0) == dw.DW_ERR_ALIAS
    # the weight gradient sizes dW and db by C*M as well
    need = dw.dwconv2d_bwd_weight_workspace_size(d)
    x, dy, dwp, db, ws = base, base + (1 << 24), base + (2 << 24), base + (3 << 24), base + (4 << 24)
    assert dw.bwd_weight_raw(d, x, dy, dwp, dwp + 8 * 9 * 4 - 4, ws, need, 0) == dw.DW_ERR_ALIAS
    assert dw.dwconv2d_query_algo(d, 2, x, dy, dwp) == dw.DW_ALGO_TILED
    d3 = dw.make_desc(1, 8, 8, 4, 3, 3, multiplier=3)
    assert dw.dwconv2d_query_algo(d3, 2, x, dy, dwp) == dw.DW_ALGO_DIRECT


def test_half_activation_host_checks(lib):
    # 16-bit activations: buffer sizes use 2-byte elements (x and y 512 B here)
    base = 1 << 40
    w = base + (1 << 20)
    for at in (dw.DW_F16, dw.DW_BF16):
        d = dw.make_desc(1, 8, 8, 4, 3, 3)
        d.atype = at
        assert dw.dwconv2d_query_algo(d, 0, base, w, base + 512) > 0        # adjacent: fine
        assert dw.fwd_raw(d, base, w, None, base + 510, 0) == dw.DW_ERR_ALIAS
        # C = 4 rows are 8 bytes: no 16-byte TMA rows, so the direct kernel
        assert dw.dwconv2d_query_algo(d, 0, base, w, base + 512) == dw.DW_ALGO_DIRECT
        d8 = dw.make_desc(1, 8, 8, 8, 3, 3)
        d8.atype = at
        assert dw.dwconv2d_query_algo(d8, 0, base, w, base + 1024) == dw.DW_ALGO_TILED
        assert dw.dwconv2d_query_algo(d8, 2, base, base + 4096, w) == dw.DW_ALGO_TILED
        dn = dw.make_desc(1, 8, 8, 8, 3, 3, layout="nchw")   # W = 8: 16-byte rows
        dn.atype = at
        assert dw.dwconv2d_query_algo(dn, 0, base, w, base + 1024) == dw.DW_ALGO_TILED
        dn4 = dw.make_desc(1, 8, 12, 8, 3, 3, layout="nchw")  # W = 12: 24-byte rows
        dn4.atype = at
        assert dw.dwconv2d_query_algo(dn4, 0, base, w, base + 4096) == dw.DW_ALGO_DIRECT


def test_selftest_rejects_bad_arguments(lib):
    # validation only: nothing is launched for these
    for mode, limit in ((2, 1000), (-1, 1000), (0, 0), (1, 2_000_000)):
        assert dw.selftest_wait_timeout_raw(mode, limit, 0) == dw.DW_ERR_INVALID_ARG


def test_query_algo_multiplier_and_16bit_tiles(lib):
    """Which family the multiplier and 16-bit calls run (dry-run dispatch):
    the NHWC and NCHW multiplier tiles for every activation type, the
    16-bit NCHW weight gradients, and the shapes that stay direct."""
    T, D = dw.DW_ALGO_TILED, dw.DW_ALGO_DIRECT
    base = 1 << 40
    ins, w_, out = base, base + (1 << 34), base + (2 << 34)   # far apart: no aliasing

    def qa(desc, op, atype=dw.DW_F32):
        desc.atype = atype
        if op == 2:   # (x, dy, dW)
            return dw.dwconv2d_query_algo(desc, 2, ins, out, w_)
        return dw.dwconv2d_query_algo(desc, op, ins, w_, out)

    for at in (dw.DW_F32, dw.DW_F16, dw.DW_BF16):
        # NHWC multiplier 2 and 4: forward, input gradient (stride 1 and 2), weight gradient
        for m in (2, 4):
            for s in (1, 2):
                d = dw.make_desc(2, 32, 32, 16, 3, 3, stride=s, multiplier=m)
                assert qa(d, 0, at) == T and qa(d, 1, at) == T and qa(d, 2, at) == T, (at, m, s)
        assert qa(dw.make_desc(2, 32, 32, 16, 5, 5, multiplier=2), 0, at) == T
        assert qa(dw.make_desc(2, 32, 32, 16, 3, 3, multiplier=3), 0, at) == D
        # NCHW multiplier: forward fan-out / one plane per tile, summed-plane input gradient
        for kh, m in ((3, 2), (3, 4), (5, 2), (7, 2)):
            d = dw.make_desc(2, 32, 32, 16, kh, kh, multiplier=m, layout="nchw")
            assert qa(d, 0, at) == T and qa(d, 1, at) == T and qa(d, 2, at) == T, (at, kh, m)
        d = dw.make_desc(2, 32, 32, 16, 5, 5, multiplier=4, layout="nchw")
        assert qa(d, 0, at) == T and qa(d, 1, at) == D
        d = dw.make_desc(2, 32, 32, 16, 3, 3, stride=2, multiplier=2, layout="nchw")
        assert qa(d, 0, at) == T and qa(d, 1, at) == T   # strided: M dy planes per box
        d = dw.make_desc(2, 32, 32, 16, 3, 3, stride=2, multiplier=4, layout="nchw")
        assert qa(d, 1, at) == D
        # NCHW weight gradients, 2-D and 1 x kW, every activation type
        assert qa(dw.make_desc(2, 16, 32, 32, 3, 3, layout="nchw"), 2, at) == T
        assert qa(dw.make_desc(2, 16, 32, 32, 3, 3, stride=2, layout="nchw"), 2, at) == T
        assert qa(dw.make_desc(2, 1, 64, 32, 1, 31, layout="nchw"), 2, at) == T
    # 16-bit NCHW rows must be 16-byte multiples: W = 36 is for float32 only
    assert qa(dw.make_desc(2, 16, 36, 32, 3, 3, layout="nchw"), 2, dw.DW_F32) == T
    assert qa(dw.make_desc(2, 16, 36, 32, 3, 3, layout="nchw"), 2, dw.DW_F16) == D
    assert qa(dw.make_desc(2, 1, 36, 32, 1, 15, layout="nchw"), 2, dw.DW_BF16) == D
