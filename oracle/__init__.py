"""Float64 CPU oracle for depthwise 2-D convolution (forward, input gradient,
weight and bias gradients).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the CPU
(reference / cpu_baseline) legs of ``bench.py`` may import this package; the
product path never does.  The arithmetic lives in ``dw_oracle.c`` (plain C
loops, float64); this module only compiles it with gcc and marshals numpy
arrays through ctypes.  Nothing here is shared with the CUDA library.

Source of every definition: page "LeanMlir Proofs/Architectures/Depthwise"
(lean.brettkoonce.com), sections "Depthwise conv2d forward", "Closed-form
input gradient ... direct formula", "Depthwise conv input-VJP", "Depthwise
weight-VJP", "Depthwise bias gradient - closed-form formula", "Stride-2 SAME
depthwise conv" and "Stride-2 XLA-SAME depthwise conv" with their VJP
sections.  Readings where
the page leaves a step open (SAME at stride > 1, bias dtype, batch axis,
layouts) are documented in ``dw_oracle.c``.

The fused forward epilogue (``bn_act``, ``fwd_bn_act``) follows the same
page's section on the MLIR lowering, which names a depthwise conv + batch-norm
emitter; it is read as inference-mode batch normalisation with running
statistics followed by an optional activation (see ``dw_oracle.c``).

Parity status: every function here is pinned by tests/test_oracle_pins.py
(hand-derived golden values, dense grouped-conv library routine, adjoint
identity, decimation identities, closed forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dw_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdw_oracle.so")
_lib = None

LAYOUTS = {"nhwc": 0, "nchw": 1}


def build(force: bool = False) -> str:
    """Compile dw_oracle.c into oracle/libdw_oracle.so (gcc, -O2, OpenMP).

    Floating-point contraction is disabled so every multiply and add rounds
    to double exactly as written in the source.
    """
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    i64, p_i64 = ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)
    p_f64 = ctypes.POINTER(ctypes.c_double)
    lib.dwo_out_extent.restype = i64
    lib.dwo_out_extent.argtypes = [i64] * 6
    lib.dwo_same_pads.restype = None
    lib.dwo_same_pads.argtypes = [i64, i64, i64, i64, p_i64, p_i64]
    lib.dwo_num_threads.restype = ctypes.c_int
    lib.dwo_num_threads.argtypes = []
    lib.dwo_fwd.restype = None
    lib.dwo_fwd.argtypes = [p_i64, p_f64, p_f64, p_f64, p_f64]
    lib.dwo_bwd_input.restype = None
    lib.dwo_bwd_input.argtypes = [p_i64, p_f64, p_f64, p_f64]
    lib.dwo_fwd_at.restype = None
    lib.dwo_fwd_at.argtypes = [p_i64, p_f64, p_f64, p_f64, i64, p_i64, p_f64]
    lib.dwo_bwd_weight.restype = None
    lib.dwo_bwd_weight.argtypes = [p_i64, p_f64, p_f64, p_f64, p_f64]
    lib.dwo_bwd_input_at.restype = None
    lib.dwo_bwd_input_at.argtypes = [p_i64, p_f64, p_f64, i64, p_i64, p_f64]
    lib.dwo_bn_act.restype = None
    lib.dwo_bn_act.argtypes = [i64, p_f64, p_i64, p_f64, p_f64, p_f64, p_f64,
                               ctypes.c_double, i64, p_f64]
    _lib = lib
    return lib


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().dwo_num_threads())


def out_extent(n_in: int, k: int, s: int, d: int, lo: int, hi: int) -> int:
    return int(_load().dwo_out_extent(n_in, k, s, d, lo, hi))


def same_pads(n_in: int, k: int, s: int, d: int) -> tuple[int, int]:
    lo, hi = ctypes.c_int64(), ctypes.c_int64()
    _load().dwo_same_pads(n_in, k, s, d, ctypes.byref(lo), ctypes.byref(hi))
    return int(lo.value), int(hi.value)


def _pair(v):
    return (int(v), int(v)) if np.isscalar(v) else (int(v[0]), int(v[1]))


def resolve_pads(H, W, kH, kW, stride=1, dilation=1, padding="same"):
    """(pt, pb, pl, pr) for padding "same" (XLA rule) or explicit.

    Explicit padding is an int (all sides), a pair (vertical, horizontal) or a
    4-tuple (top, bottom, left, right).
    """
    sh, sw = _pair(stride)
    dh, dw = _pair(dilation)
    if isinstance(padding, str):
        if padding.lower() != "same":
            raise ValueError(f"unknown padding mode {padding!r}")
        pt, pb = same_pads(H, kH, sh, dh)
        pl, pr = same_pads(W, kW, sw, dw)
        return pt, pb, pl, pr
    if np.isscalar(padding):
        p = int(padding)
        return p, p, p, p
    padding = tuple(int(v) for v in padding)
    if len(padding) == 2:
        return padding[0], padding[0], padding[1], padding[1]
    if len(padding) == 4:
        return padding
    raise ValueError(f"bad padding {padding!r}")


def problem(shape, kH, kW, stride=1, dilation=1, padding="same", layout="nhwc", multiplier=1):
    """int64[16] problem vector from the input activation shape in `layout`
    order; `multiplier` M output channels per input channel (C*M in all)."""
    layout = layout.lower()
    if layout == "nhwc":
        N, H, W, C = shape
    elif layout == "nchw":
        N, C, H, W = shape
    else:
        raise ValueError(layout)
    sh, sw = _pair(stride)
    dh, dw = _pair(dilation)
    pt, pb, pl, pr = resolve_pads(H, W, kH, kW, stride, dilation, padding)
    if int(multiplier) < 1:
        raise ValueError("multiplier must be >= 1")
    return np.array([N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr,
                     LAYOUTS[layout], int(multiplier)], dtype=np.int64)


def out_channels(prob) -> int:
    return int(prob[3]) * int(prob[15])


def out_shape(prob) -> tuple[int, ...]:
    N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr, lay, M = (int(v) for v in prob)
    Ho = out_extent(H, kH, sh, dh, pt, pb)
    Wo = out_extent(W, kW, sw, dw, pl, pr)
    return (N, Ho, Wo, C * M) if lay == 0 else (N, C * M, Ho, Wo)


def in_shape(prob) -> tuple[int, ...]:
    N, H, W, C = (int(v) for v in prob[:4])
    return (N, H, W, C) if int(prob[14]) == 0 else (N, C, H, W)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, ty=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ty))


def _weights(w, prob):
    kH, kW = int(prob[4]), int(prob[5])
    return _f64(w).reshape(out_channels(prob), kH, kW)


def fwd(prob, x, w, b=None):
    """y = depthwise forward (float64) for problem vector `prob`."""
    prob = np.ascontiguousarray(prob, dtype=np.int64)
    x = _f64(x).reshape(in_shape(prob))
    w = _weights(w, prob)
    bb = None if b is None else _f64(b).reshape(out_channels(prob))
    y = np.empty(out_shape(prob), dtype=np.float64)
    _load().dwo_fwd(_ptr(prob, ctypes.c_int64), _ptr(x), _ptr(w),
                    None if bb is None else _ptr(bb), _ptr(y))
    return y


def bwd_input(prob, dy, w):
    """dx = transpose of the forward's linear part applied to dy (float64)."""
    prob = np.ascontiguousarray(prob, dtype=np.int64)
    dy = _f64(dy).reshape(out_shape(prob))
    w = _weights(w, prob)
    dx = np.empty(in_shape(prob), dtype=np.float64)
    _load().dwo_bwd_input(_ptr(prob, ctypes.c_int64), _ptr(dy), _ptr(w), _ptr(dx))
    return dx


def fwd_at(prob, x, w, b, flat_idx):
    """Forward output at the given flat indices of y (layout order)."""
    prob = np.ascontiguousarray(prob, dtype=np.int64)
    x = _f64(x).reshape(in_shape(prob))
    w = _weights(w, prob)
    bb = None if b is None else _f64(b).reshape(out_channels(prob))
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    out = np.empty(idx.shape[0], dtype=np.float64)
    _load().dwo_fwd_at(_ptr(prob, ctypes.c_int64), _ptr(x), _ptr(w),
                       None if bb is None else _ptr(bb), idx.shape[0],
                       _ptr(idx, ctypes.c_int64), _ptr(out))
    return out


def bwd_input_at(prob, dy, w, flat_idx):
    """Input gradient at the given flat indices of dx, by the direct formula."""
    prob = np.ascontiguousarray(prob, dtype=np.int64)
    dy = _f64(dy).reshape(out_shape(prob))
    w = _weights(w, prob)
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    out = np.empty(idx.shape[0], dtype=np.float64)
    _load().dwo_bwd_input_at(_ptr(prob, ctypes.c_int64), _ptr(dy), _ptr(w),
                             idx.shape[0], _ptr(idx, ctypes.c_int64), _ptr(out))
    return out


def bwd_weight(prob, x, dy):
    """(dW [C*M,kH,kW], db [C*M]): weight and bias gradients of the forward (float64)."""
    prob = np.ascontiguousarray(prob, dtype=np.int64)
    x = _f64(x).reshape(in_shape(prob))
    dy = _f64(dy).reshape(out_shape(prob))
    C, kH, kW = out_channels(prob), int(prob[4]), int(prob[5])
    dw = np.empty((C, kH, kW), dtype=np.float64)
    db = np.empty(C, dtype=np.float64)
    _load().dwo_bwd_weight(_ptr(prob, ctypes.c_int64), _ptr(x), _ptr(dy), _ptr(dw), _ptr(db))
    return dw, db


ACTS = {"none": 0, "relu": 1, "relu6": 2, "silu": 3}


def channel_of(prob, flat_idx, out=True):
    """Channel of each flat index of y (out=True) or x, in the problem's layout."""
    idx = np.asarray(flat_idx, dtype=np.int64)
    shape = out_shape(prob) if out else in_shape(prob)
    if int(prob[14]) == 0:
        return idx % shape[3]
    return (idx // (shape[2] * shape[3])) % shape[1]


def bn_act(prob, z, flat_idx=None, bn=None, act="none"):
    """Fused epilogue applied to forward values z (float64).

    z holds the forward output at the flat y indices `flat_idx` (all of y, in
    layout order, when None).  bn = (gamma, beta, mean, var, eps) or None.
    """
    z = _f64(z)
    flat = z.reshape(-1)
    idx = np.arange(flat.size, dtype=np.int64) if flat_idx is None else \
        np.ascontiguousarray(flat_idx, dtype=np.int64)
    ch = np.ascontiguousarray(channel_of(prob, idx), dtype=np.int64)
    out = np.empty_like(flat)
    C = out_channels(prob)
    if bn is None:
        g = be = mu = var = None
        eps = 0.0
    else:
        g, be, mu, var = (_f64(v).reshape(C) for v in bn[:4])
        eps = float(bn[4])
    _load().dwo_bn_act(flat.size, _ptr(flat), _ptr(ch, ctypes.c_int64),
                       None if g is None else _ptr(g), None if g is None else _ptr(be),
                       None if g is None else _ptr(mu), None if g is None else _ptr(var),
                       eps, ACTS[act], _ptr(out))
    return out.reshape(z.shape)


def fwd_bn_act(prob, x, w, b=None, bn=None, act="none"):
    """act(batch_norm(forward(x)))  (float64); bn = (gamma, beta, mean, var, eps) or None."""
    return bn_act(prob, fwd(prob, x, w, b), None, bn, act)
