"""Depthwise 2-D convolution (forward and input gradient) for NVIDIA B200.

The compute lives in libdwconv2d.so (hand-written CUDA for sm_100a, C ABI in
include/dwconv2d.h); this package is its thin Python binding.  Build the
library with ``python -m depthwise_convolution_fwd_b200.build``.
"""
from .dwconv2d import (  # noqa: F401
    DW_ACT_NONE, DW_ACT_RELU, DW_ACT_RELU6, DW_ACT_SILU, DW_ALGO_AUTO, DW_ALGO_DIRECT, DW_ALGO_TILED, DW_ERR_ALIAS, DW_ERR_CUDA,
    DW_ERR_DEVICE_TIMEOUT, DW_ERR_INVALID_ARG, DW_ERR_TOO_LARGE, DW_NOALLOC_SCRATCH_BYTES, DW_ERR_UNSUPPORTED, DW_BF16, DW_F16, DW_F32, DW_NCHW,
    DW_NHWC, DW_OK, DW_PAD_EXPLICIT, DW_PAD_SAME, EXPORTS, DwDesc, DwError, bwd_input_raw,
    bwd_weight_noalloc_raw, bwd_weight_raw, dwconv2d_bwd_input, dwconv2d_bwd_weight, dwconv2d_bwd_weight_workspace_size,
    dwconv2d_fwd, dwconv2d_fwd_bn_act, dwconv2d_out_shape, fwd_bn_act_raw, dwconv2d_query_algo,
    dwconv2d_resolved_pads, dwconv2d_take_device_error, dwconv2d_version, fwd_raw, lib,
    library_path, make_desc, selftest_wait_timeout_raw, status_string,
)
