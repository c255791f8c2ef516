"""Thin Python binding over libdwconv2d (include/dwconv2d.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libdwconv2d.so.  PyTorch supplies device memory and the stream.
There is no CPU or PyTorch fallback: if the library is missing or a tensor is
not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple, Union

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdwconv2d.so")
_lib = None

(DW_OK, DW_ERR_INVALID_ARG, DW_ERR_UNSUPPORTED, DW_ERR_ALIAS, DW_ERR_CUDA,
 DW_ERR_DEVICE_TIMEOUT, DW_ERR_TOO_LARGE) = range(7)
DW_NOALLOC_SCRATCH_BYTES = 16 << 20
DW_NHWC, DW_NCHW = 0, 1
DW_F32, DW_F16, DW_BF16 = 0, 1, 2
DW_PAD_EXPLICIT, DW_PAD_SAME = 0, 1
DW_ALGO_AUTO, DW_ALGO_DIRECT, DW_ALGO_TILED = 0, 1, 2
DW_ACT_NONE, DW_ACT_RELU, DW_ACT_RELU6, DW_ACT_SILU = 0, 1, 2, 3

_LAYOUTS = {"nhwc": DW_NHWC, "nchw": DW_NCHW}
_ALGOS = {"auto": DW_ALGO_AUTO, "direct": DW_ALGO_DIRECT, "tiled": DW_ALGO_TILED}
_ACTS = {"none": DW_ACT_NONE, "relu": DW_ACT_RELU, "relu6": DW_ACT_RELU6, "silu": DW_ACT_SILU}

# Every symbol include/dwconv2d.h declares.
EXPORTS = ("dwconv2d_out_shape", "dwconv2d_resolved_pads", "dwconv2d_fwd", "dwconv2d_fwd_bn_act",
           "dwconv2d_bwd_input", "dwconv2d_bwd_weight", "dwconv2d_bwd_weight_workspace_size",
           "dwconv2d_bwd_weight_noalloc",
           "dwconv2d_query_algo", "dwconv2d_take_device_error", "dwconv2d_status_string",
           "dwconv2d_selftest_wait_timeout",
           "dwconv2d_version")


class DwDesc(ctypes.Structure):
    """Mirror of dw_desc_t."""
    _fields_ = [("N", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
                ("C", ctypes.c_int64), ("kH", ctypes.c_int32), ("kW", ctypes.c_int32),
                ("stride_h", ctypes.c_int32), ("stride_w", ctypes.c_int32),
                ("dil_h", ctypes.c_int32), ("dil_w", ctypes.c_int32),
                ("pad_mode", ctypes.c_int32), ("pad_top", ctypes.c_int32),
                ("pad_bottom", ctypes.c_int32), ("pad_left", ctypes.c_int32),
                ("pad_right", ctypes.c_int32), ("layout", ctypes.c_int32),
                ("wtype", ctypes.c_int32), ("algo", ctypes.c_int32),
                ("multiplier", ctypes.c_int32), ("atype", ctypes.c_int32)]


class DwError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded libdwconv2d.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"libdwconv2d.so not found at {_LIB_PATH}; build it with "
            "`python -m depthwise_convolution_fwd_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    P = ctypes.POINTER
    i32, i64, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    L.dwconv2d_out_shape.restype = i32
    L.dwconv2d_out_shape.argtypes = [P(DwDesc), P(i64), P(i64)]
    L.dwconv2d_resolved_pads.restype = i32
    L.dwconv2d_resolved_pads.argtypes = [P(DwDesc), P(i32)]
    L.dwconv2d_fwd.restype = i32
    L.dwconv2d_fwd.argtypes = [P(DwDesc), vp, vp, vp, vp, vp]
    L.dwconv2d_bwd_input.restype = i32
    L.dwconv2d_bwd_input.argtypes = [P(DwDesc), vp, vp, vp, vp]
    L.dwconv2d_fwd_bn_act.restype = i32
    L.dwconv2d_fwd_bn_act.argtypes = [P(DwDesc), vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, i32,
                                      vp, vp]
    L.dwconv2d_bwd_weight.restype = i32
    L.dwconv2d_bwd_weight.argtypes = [P(DwDesc), vp, vp, vp, vp, vp, ctypes.c_uint64, vp]
    L.dwconv2d_bwd_weight_noalloc.restype = i32
    L.dwconv2d_bwd_weight_noalloc.argtypes = [P(DwDesc), vp, vp, vp, vp, vp]
    L.dwconv2d_bwd_weight_workspace_size.restype = i32
    L.dwconv2d_bwd_weight_workspace_size.argtypes = [P(DwDesc), P(ctypes.c_uint64)]
    L.dwconv2d_query_algo.restype = i32
    L.dwconv2d_query_algo.argtypes = [P(DwDesc), i32, vp, vp, vp]
    L.dwconv2d_take_device_error.restype = i32
    L.dwconv2d_take_device_error.argtypes = [P(i32)]
    L.dwconv2d_selftest_wait_timeout.restype = i32
    L.dwconv2d_selftest_wait_timeout.argtypes = [i32, ctypes.c_uint32, vp]
    L.dwconv2d_status_string.restype = ctypes.c_char_p
    L.dwconv2d_status_string.argtypes = [i32]
    L.dwconv2d_version.restype = i32
    L.dwconv2d_version.argtypes = []
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().dwconv2d_status_string(int(status)).decode()


def _pair(v) -> Tuple[int, int]:
    if isinstance(v, (tuple, list)):
        return int(v[0]), int(v[1])
    return int(v), int(v)


def make_desc(N: int, H: int, W: int, C: int, kH: int, kW: int, *, stride=1, dilation=1,
              padding: Union[str, int, Sequence[int]] = "same", layout: str = "nhwc",
              wtype: str = "f32", algo: str = "auto", multiplier: int = 1,
              atype: str = "f32") -> DwDesc:
    """Descriptor for input extents N,H,W,C.  padding: "same" (XLA rule), an
    int, a (vertical, horizontal) pair or (top, bottom, left, right);
    multiplier: output channels per input channel (C*multiplier in all);
    atype: activation element type "f32", "f16" or "bf16"."""
    d = DwDesc()
    d.N, d.H, d.W, d.C = int(N), int(H), int(W), int(C)
    d.kH, d.kW = int(kH), int(kW)
    d.stride_h, d.stride_w = _pair(stride)
    d.dil_h, d.dil_w = _pair(dilation)
    if isinstance(padding, str):
        if padding.lower() != "same":
            raise ValueError(f"unknown padding {padding!r}")
        d.pad_mode = DW_PAD_SAME
    else:
        d.pad_mode = DW_PAD_EXPLICIT
        if isinstance(padding, int):
            pads = (padding,) * 4
        elif len(padding) == 2:
            pads = (padding[0], padding[0], padding[1], padding[1])
        else:
            pads = tuple(padding)
        d.pad_top, d.pad_bottom, d.pad_left, d.pad_right = (int(v) for v in pads)
    d.layout = _LAYOUTS[layout.lower()]
    d.wtype = {"f32": DW_F32, "f16": DW_F16}[wtype]
    d.algo = _ALGOS[algo]
    d.multiplier = int(multiplier)
    d.atype = {"f32": DW_F32, "f16": DW_F16, "bf16": DW_BF16}[atype]
    return d


def dwconv2d_out_shape(desc: DwDesc) -> Tuple[int, int]:
    ho, wo = ctypes.c_int64(), ctypes.c_int64()
    st = lib().dwconv2d_out_shape(ctypes.byref(desc), ctypes.byref(ho), ctypes.byref(wo))
    if st != DW_OK:
        raise DwError(st, "dwconv2d_out_shape")
    return int(ho.value), int(wo.value)


def dwconv2d_resolved_pads(desc: DwDesc) -> Tuple[int, int, int, int]:
    pads = (ctypes.c_int32 * 4)()
    st = lib().dwconv2d_resolved_pads(ctypes.byref(desc), pads)
    if st != DW_OK:
        raise DwError(st, "dwconv2d_resolved_pads")
    return tuple(int(v) for v in pads)


def dwconv2d_query_algo(desc: DwDesc, op: int, inp: int, w: int, out: int) -> int:
    return int(lib().dwconv2d_query_algo(ctypes.byref(desc), int(op), inp, w, out))


def dwconv2d_take_device_error() -> int:
    code = ctypes.c_int32()
    st = lib().dwconv2d_take_device_error(ctypes.byref(code))
    if st != DW_OK:
        raise DwError(st, "dwconv2d_take_device_error")
    return int(code.value)


def selftest_wait_timeout_raw(mode: int, limit_us: int, stream: int) -> int:
    """dwconv2d_selftest_wait_timeout: a kernel whose bounded wait runs out
    (mode 0) or is aborted by another warp (mode 1); returns the status.  The
    device error word then holds DW_ERR_DEVICE_TIMEOUT."""
    return int(lib().dwconv2d_selftest_wait_timeout(int(mode), int(limit_us), stream or None))


def dwconv2d_version() -> int:
    return int(lib().dwconv2d_version())


# ------------------------------------------------------- raw pointer calls --

def fwd_raw(desc: DwDesc, x_ptr: int, w_ptr: int, b_ptr: Optional[int], y_ptr: int,
            stream: int) -> int:
    """dwconv2d_fwd on raw device pointers; returns the status."""
    return int(lib().dwconv2d_fwd(ctypes.byref(desc), x_ptr, w_ptr, b_ptr or None, y_ptr,
                                  stream or None))


def fwd_bn_act_raw(desc: DwDesc, x_ptr: int, w_ptr: int, b_ptr: Optional[int],
                   bn_ptrs: Optional[Sequence[int]], eps: float, act: int, y_ptr: int,
                   stream: int) -> int:
    """dwconv2d_fwd_bn_act on raw device pointers (bn_ptrs = gamma, beta, mean,
    var or None); returns the status."""
    g, be, mu, var = bn_ptrs if bn_ptrs is not None else (None, None, None, None)
    return int(lib().dwconv2d_fwd_bn_act(ctypes.byref(desc), x_ptr, w_ptr, b_ptr or None,
                                         g or None, be or None, mu or None, var or None,
                                         float(eps), int(act), y_ptr, stream or None))


def bwd_input_raw(desc: DwDesc, dy_ptr: int, w_ptr: int, dx_ptr: int, stream: int) -> int:
    """dwconv2d_bwd_input on raw device pointers; returns the status."""
    return int(lib().dwconv2d_bwd_input(ctypes.byref(desc), dy_ptr, w_ptr, dx_ptr,
                                        stream or None))


def bwd_weight_raw(desc: DwDesc, x_ptr: int, dy_ptr: int, dw_ptr: int, db_ptr: Optional[int],
                   ws_ptr: int, ws_bytes: int, stream: int) -> int:
    """dwconv2d_bwd_weight on raw device pointers; returns the status."""
    return int(lib().dwconv2d_bwd_weight(ctypes.byref(desc), x_ptr, dy_ptr, dw_ptr, db_ptr or None,
                                         ws_ptr, int(ws_bytes), stream or None))


def bwd_weight_noalloc_raw(desc: DwDesc, x_ptr: int, dy_ptr: int, dw_ptr: int,
                           db_ptr: Optional[int], stream: int) -> int:
    """dwconv2d_bwd_weight_noalloc on raw device pointers; returns the status.
    For callers that cannot allocate device memory: the scratch is a fixed
    array inside the library (see include/dwconv2d.h)."""
    return int(lib().dwconv2d_bwd_weight_noalloc(ctypes.byref(desc), x_ptr, dy_ptr, dw_ptr,
                                                 db_ptr or None, stream or None))


def dwconv2d_bwd_weight_workspace_size(desc: DwDesc) -> int:
    n = ctypes.c_uint64()
    st = lib().dwconv2d_bwd_weight_workspace_size(ctypes.byref(desc), ctypes.byref(n))
    if st != DW_OK:
        raise DwError(st, "dwconv2d_bwd_weight_workspace_size")
    return int(n.value)


# ------------------------------------------------------------ tensor calls --

_ATYPES = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}


def _check_act(t: torch.Tensor, name: str, dtype: Optional[torch.dtype] = None):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in _ATYPES:
        raise TypeError(f"{name} must be float32, float16 or bfloat16, got {t.dtype}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} like the other activations, got {t.dtype}")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 4-D tensor")


def _weights(w: torch.Tensor, C: int, device) -> Tuple[torch.Tensor, int, int, str]:
    """w: [C,kH,kW] or [C,1,kH,kW] where C counts the OUTPUT channels."""
    if not isinstance(w, torch.Tensor) or w.device != device:
        raise TypeError("w must be a CUDA tensor on the activations' device")
    if w.dim() == 4:
        if w.shape[0] != C or w.shape[1] != 1:
            raise ValueError(f"w must be [C,1,kH,kW] with C={C}, got {tuple(w.shape)}")
        kH, kW = int(w.shape[2]), int(w.shape[3])
    elif w.dim() == 3:
        if w.shape[0] != C:
            raise ValueError(f"w must be [C,kH,kW] with C={C}, got {tuple(w.shape)}")
        kH, kW = int(w.shape[1]), int(w.shape[2])
    else:
        raise ValueError("w must be [C,kH,kW] or [C,1,kH,kW]")
    if not w.is_contiguous():
        raise ValueError("w must be contiguous")
    if w.dtype == torch.float32:
        wt = "f32"
    elif w.dtype == torch.float16:
        wt = "f16"
    else:
        raise TypeError(f"w must be float32 or float16, got {w.dtype}")
    return w, kH, kW, wt


def _out_channels(w: torch.Tensor, C: int) -> Tuple[int, int]:
    """(C*M, M) from the filter's leading extent: M filters per input channel."""
    if not isinstance(w, torch.Tensor) or w.dim() < 1:
        raise TypeError("w must be a tensor")
    Co = int(w.shape[0])
    if Co < C or Co % C != 0:
        raise ValueError(f"w must have C*multiplier rows for C={C}, got {Co}")
    return Co, Co // C


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def dwconv2d_fwd(x: torch.Tensor, w: torch.Tensor, b: Optional[torch.Tensor] = None, *,
                 stride=1, dilation=1, padding="same", layout: str = "nhwc",
                 algo: str = "auto", out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = depthwise conv2d forward of x (layout "nhwc" [N,H,W,C] or "nchw"
    [N,C,H,W]) with weights w [C,kH,kW] (float32 or float16) and bias b [C]."""
    _check_act(x, "x")
    if layout.lower() == "nhwc":
        N, H, W, C = x.shape
    else:
        N, C, H, W = x.shape
    Co, M = _out_channels(w, C)
    w, kH, kW, wt = _weights(w, Co, x.device)
    if b is not None:
        if b.device != x.device or b.dtype != torch.float32 or b.numel() != Co or not b.is_contiguous():
            raise ValueError("b must be a contiguous float32 CUDA tensor of C*multiplier elements")
    desc = make_desc(N, H, W, C, kH, kW, stride=stride, dilation=dilation, padding=padding,
                     layout=layout, wtype=wt, algo=algo, multiplier=M, atype=_ATYPES[x.dtype])
    Ho, Wo = dwconv2d_out_shape(desc)
    shape = (N, Ho, Wo, Co) if desc.layout == DW_NHWC else (N, Co, Ho, Wo)
    if out is None:
        out = torch.empty(shape, device=x.device, dtype=x.dtype)
    else:
        _check_act(out, "out", x.dtype)
        if tuple(out.shape) != shape or out.device != x.device:
            raise ValueError(f"out must have shape {shape} on {x.device}")
    with torch.cuda.device(x.device):
        st = fwd_raw(desc, x.data_ptr(), w.data_ptr(), None if b is None else b.data_ptr(),
                     out.data_ptr(), _stream_ptr(x.device))
    if st != DW_OK:
        raise DwError(st, "dwconv2d_fwd")
    return out


def dwconv2d_fwd_bn_act(x: torch.Tensor, w: torch.Tensor, b: Optional[torch.Tensor] = None,
                        bn: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor,
                                           torch.Tensor, float]] = None,
                        act: str = "none", *, stride=1, dilation=1, padding="same",
                        layout: str = "nhwc", algo: str = "auto",
                        out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = act(batch_norm(depthwise conv2d forward(x) + b)) in one kernel.

    bn = (gamma, beta, running_mean, running_var, eps) with [C] float32 CUDA
    tensors (inference-mode statistics) or None; act in "none", "relu",
    "relu6", "silu".  Other arguments as for dwconv2d_fwd."""
    _check_act(x, "x")
    if layout.lower() == "nhwc":
        N, H, W, C = x.shape
    else:
        N, C, H, W = x.shape
    Co, M = _out_channels(w, C)
    w, kH, kW, wt = _weights(w, Co, x.device)
    if b is not None:
        if b.device != x.device or b.dtype != torch.float32 or b.numel() != Co or not b.is_contiguous():
            raise ValueError("b must be a contiguous float32 CUDA tensor of C*multiplier elements")
    ptrs, eps = None, 0.0
    if bn is not None:
        if len(bn) != 5:
            raise ValueError("bn must be (gamma, beta, running_mean, running_var, eps)")
        for t in bn[:4]:
            if (not isinstance(t, torch.Tensor) or t.device != x.device or t.dtype != torch.float32
                    or t.numel() != Co or not t.is_contiguous()):
                raise ValueError("batch-norm statistics must be contiguous float32 CUDA tensors of "
                                 "C*multiplier elements")
        ptrs = [t.data_ptr() for t in bn[:4]]
        eps = float(bn[4])
    if act not in _ACTS:
        raise ValueError(f"act must be one of {sorted(_ACTS)}")
    desc = make_desc(N, H, W, C, kH, kW, stride=stride, dilation=dilation, padding=padding,
                     layout=layout, wtype=wt, algo=algo, multiplier=M, atype=_ATYPES[x.dtype])
    Ho, Wo = dwconv2d_out_shape(desc)
    shape = (N, Ho, Wo, Co) if desc.layout == DW_NHWC else (N, Co, Ho, Wo)
    if out is None:
        out = torch.empty(shape, device=x.device, dtype=x.dtype)
    else:
        _check_act(out, "out", x.dtype)
        if tuple(out.shape) != shape or out.device != x.device:
            raise ValueError(f"out must have shape {shape} on {x.device}")
    with torch.cuda.device(x.device):
        st = fwd_bn_act_raw(desc, x.data_ptr(), w.data_ptr(), None if b is None else b.data_ptr(),
                            ptrs, eps, _ACTS[act], out.data_ptr(), _stream_ptr(x.device))
    if st != DW_OK:
        raise DwError(st, "dwconv2d_fwd_bn_act")
    return out


def dwconv2d_bwd_input(dy: torch.Tensor, w: torch.Tensor, input_hw: Tuple[int, int], *,
                       stride=1, dilation=1, padding="same", layout: str = "nhwc",
                       algo: str = "auto", out: Optional[torch.Tensor] = None,
                       multiplier: int = 1) -> torch.Tensor:
    """dx = input gradient of the forward whose input had spatial extents
    input_hw = (H, W), given the output cotangent dy (C*multiplier channels)."""
    _check_act(dy, "dy")
    H, W = (int(v) for v in input_hw)
    if layout.lower() == "nhwc":
        N, Ho, Wo, Co = dy.shape
    else:
        N, Co, Ho, Wo = dy.shape
    M = int(multiplier)
    if M < 1 or Co % M != 0:
        raise ValueError(f"dy's {Co} channels are not a multiple of multiplier {M}")
    C = Co // M
    w, kH, kW, wt = _weights(w, Co, dy.device)
    desc = make_desc(N, H, W, C, kH, kW, stride=stride, dilation=dilation, padding=padding,
                     layout=layout, wtype=wt, algo=algo, multiplier=M, atype=_ATYPES[dy.dtype])
    if dwconv2d_out_shape(desc) != (Ho, Wo):
        raise ValueError(f"dy spatial extents {(Ho, Wo)} do not match the forward's "
                         f"{dwconv2d_out_shape(desc)}")
    shape = (N, H, W, C) if desc.layout == DW_NHWC else (N, C, H, W)
    if out is None:
        out = torch.empty(shape, device=dy.device, dtype=dy.dtype)
    else:
        _check_act(out, "out", dy.dtype)
        if tuple(out.shape) != shape or out.device != dy.device:
            raise ValueError(f"out must have shape {shape} on {dy.device}")
    with torch.cuda.device(dy.device):
        st = bwd_input_raw(desc, dy.data_ptr(), w.data_ptr(), out.data_ptr(),
                           _stream_ptr(dy.device))
    if st != DW_OK:
        raise DwError(st, "dwconv2d_bwd_input")
    return out


def dwconv2d_bwd_weight(x: torch.Tensor, dy: torch.Tensor, kernel_hw: Tuple[int, int], *,
                        stride=1, dilation=1, padding="same", layout: str = "nhwc",
                        algo: str = "auto", bias: bool = True,
                        dw: Optional[torch.Tensor] = None, db: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None):
    """(dW [C*M,kH,kW], db [C*M] or None): weight and bias gradients of the
    forward with input x (C channels) and output cotangent dy (C*M channels;
    M, the channel multiplier, is read off dy).  `workspace` (a CUDA byte
    tensor of at least dwconv2d_bwd_weight_workspace_size bytes) is allocated
    when not given."""
    _check_act(x, "x")
    _check_act(dy, "dy", x.dtype)
    if dy.device != x.device:
        raise ValueError("x and dy must be on the same device")
    kH, kW = (int(v) for v in kernel_hw)
    if layout.lower() == "nhwc":
        N, H, W, C = x.shape
    else:
        N, C, H, W = x.shape
    Co = int(dy.shape[3] if layout.lower() == "nhwc" else dy.shape[1])
    if Co < C or Co % C != 0:
        raise ValueError(f"dy must have C*multiplier channels for C={C}, got {Co}")
    desc = make_desc(N, H, W, C, kH, kW, stride=stride, dilation=dilation, padding=padding,
                     layout=layout, algo=algo, multiplier=Co // C, atype=_ATYPES[x.dtype])
    Ho, Wo = dwconv2d_out_shape(desc)
    want = (N, Ho, Wo, Co) if desc.layout == DW_NHWC else (N, Co, Ho, Wo)
    if tuple(dy.shape) != want:
        raise ValueError(f"dy must have shape {want}, got {tuple(dy.shape)}")
    if dw is None:
        dw = torch.empty((Co, kH, kW), device=x.device, dtype=torch.float32)
    elif dw.dtype != torch.float32 or dw.numel() != Co * kH * kW or not dw.is_contiguous():
        raise ValueError("dw must be a contiguous float32 tensor of C*multiplier*kH*kW elements")
    if bias and db is None:
        db = torch.empty((Co,), device=x.device, dtype=torch.float32)
    need = dwconv2d_bwd_weight_workspace_size(desc)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), device=x.device, dtype=torch.uint8)
    elif workspace.device != x.device or workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace must hold at least {need} bytes on {x.device}")
    with torch.cuda.device(x.device):
        st = bwd_weight_raw(desc, x.data_ptr(), dy.data_ptr(), dw.data_ptr(),
                            None if db is None else db.data_ptr(), workspace.data_ptr(),
                            workspace.numel() * workspace.element_size(), _stream_ptr(x.device))
    if st != DW_OK:
        raise DwError(st, "dwconv2d_bwd_weight")
    return dw, db
