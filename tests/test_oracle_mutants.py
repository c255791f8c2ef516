"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake (a dropped term, a wrong sign or index, a
flipped or transposed operand, an off-by-one) in a private copy of
oracle/dw_oracle.c, compiles it to a temporary directory and runs a fast
subset of the pin checks against it.  The unmodified oracle must pass them
all; every mutant must fail at least one.  Nothing here touches the real
oracle library or any GPU.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "dw_oracle.c")

MUTANTS = {
    "fwd_flipped_kernel": ("acc += xv * wt[(o * kH + kh) * kW + kw];",
                           "acc += xv * wt[(o * kH + (kH - 1 - kh)) * kW + (kW - 1 - kw)];"),
    "fwd_pad_sign": ("int64_t hi = ho * p[P_SH] + kh * p[P_DH] - p[P_PT];\n            int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];\n            double xv",
                     "int64_t hi = ho * p[P_SH] + kh * p[P_DH] + p[P_PT];\n            int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];\n            double xv"),
    "fwd_dropped_bias": ("return acc + (b ? b[o] : 0.0);", "return acc;"),
    "fwd_swapped_strides": ("int64_t hi = ho * p[P_SH] + kh * p[P_DH] - p[P_PT];\n            int64_t wi = wo * p[P_SW]",
                            "int64_t hi = ho * p[P_SW] + kh * p[P_DH] - p[P_PT];\n            int64_t wi = wo * p[P_SH]"),
    "fwd_transposed_taps": ("acc += xv * wt[(o * kH + kh) * kW + kw];",
                            "acc += xv * wt[(o * kW + kw) * kH + kh];"),
    "bwd_flipped_kernel": ("g * wt[(o * kH + kh) * kW + kw];",
                           "g * wt[(o * kH + (kH - 1 - kh)) * kW + (kW - 1 - kw)];"),
    "bwd_dropped_dilation": ("int64_t hi = ho * p[P_SH] + kh * p[P_DH] - p[P_PT];\n                                int64_t wi",
                             "int64_t hi = ho * p[P_SH] + kh - p[P_PT];\n                                int64_t wi"),
    "bwd_wrong_pad_side": ("int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];\n                                if (hi < 0",
                           "int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PR];\n                                if (hi < 0"),
    "same_odd_half_on_top": ("*lo = total / 2;\n    *hi = total - *lo;", "*hi = total / 2;\n    *lo = total - *hi;"),
    "extent_off_by_one": ("return last_reach / s + 1;", "return last_reach / s;"),
    "bwd_at_no_divisibility": ("if (kh_nat % dh != 0) continue;", ""),
    "wgrad_pad_sign": ("int64_t hi = ho * p[P_SH] + kh * p[P_DH] - p[P_PT];\n                            int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];\n                            if (hi < 0 || hi >= H || wi < 0 || wi >= W) continue;\n                            acc +=",
                       "int64_t hi = ho * p[P_SH] + kh * p[P_DH] + p[P_PT];\n                            int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];\n                            if (hi < 0 || hi >= H || wi < 0 || wi >= W) continue;\n                            acc +="),
    "wgrad_transposed_taps": ("dw[(o * kH + kh) * kW + kw] = acc;", "dw[(o * kW + kw) * kH + kh] = acc;"),
    "bwd_at_channel_mix": ("acc += dy[act_index(p, n, o, ho, wo, out_c(p), Ho, Wo)] *\n                           wt[(o * kH + kh) * kW + kw];",
                           "acc += dy[act_index(p, n, o, ho, wo, out_c(p), Ho, Wo)] *\n                           wt[(((o + 1) % out_c(p)) * kH + kh) * kW + kw];"),
    "mult_fwd_input_channel": ("int64_t c = o / p[P_MULT];  /* the one input channel output o reads */",
                               "int64_t c = o % p[P_C];"),
    "mult_bwd_first_output_only": ("for (int64_t o = c * M; o < (c + 1) * M; ++o)",
                                   "for (int64_t o = c * M; o < c * M + 1; ++o)"),
    "mult_bwd_at_first_output_only": ("for (int64_t o = c * p[P_MULT]; o < (c + 1) * p[P_MULT]; ++o)",
                                      "for (int64_t o = c * p[P_MULT]; o < c * p[P_MULT] + 1; ++o)"),
    "mult_wgrad_input_channel": ("int64_t c = o / p[P_MULT];  /* the input channel filter o reads */",
                                 "int64_t c = o % p[P_C];"),
    "bn_dropped_eps": ("(u - mean[c]) / sqrt(var[c] + eps)", "(u - mean[c]) / sqrt(var[c])"),
    "bn_mean_sign": ("(u - mean[c])", "(u + mean[c])"),
    "bn_channel_ignored": ("int64_t c = ch[i];", "int64_t c = 0;"),
    "bn_bias_after_norm": ("gamma[c] * (u - mean[c]) / sqrt(var[c] + eps) + beta[c]",
                           "gamma[c] * u / sqrt(var[c] + eps) + beta[c] - mean[c]"),
    "relu6_no_upper_clamp": ("(u > 6.0 ? 6.0 : u)", "u"),
    "silu_wrong_sign": ("u / (1.0 + exp(-u))", "u / (1.0 + exp(u))"),
}


def build_variant(tmp_path, name, patch):
    src = open(SRC).read()
    if patch is not None:
        old, new = patch
        assert src.count(old) >= 1, f"mutant {name}: pattern not found"
        src = src.replace(old, new, 1)
    c_path = tmp_path / f"{name}.c"
    c_path.write_text(src)
    so_path = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                    str(c_path), "-o", str(so_path), "-lm"], check=True)
    return str(so_path)


def run_pin_subset():
    """Fast subset of tests/test_oracle_pins.py; returns names of failed checks."""
    failed = []
    checks = [
        ("golden_orientation", lambda: [pins.test_golden_orientation(None, l) for l in ("nhwc", "nchw")]),
        ("golden_stride2", lambda: [pins.test_golden_stride2_even_and_odd_decimation(None, l) for l in ("nhwc", "nchw")]),
        ("golden_dilation", lambda: pins.test_golden_dilation(None)),
        ("golden_channels", lambda: [pins.test_golden_channels_and_asymmetric_pads(None, l) for l in ("nhwc", "nchw")]),
        ("golden_shapes", lambda: pins.test_golden_shape_pins(None)),
        ("torch_fwd", lambda: pins.test_fwd_equals_torch_conv2d(None, False)),
        ("torch_bwd", lambda: pins.test_bwd_equals_torch_autograd(None)),
        ("adjoint", lambda: pins.test_adjoint_identity(None)),
        ("sampled", lambda: pins.test_sampled_evaluators_match_full(None)),
        ("golden_wgrad", lambda: pins.test_golden_weight_gradient(None)),
        ("wgrad_linearity", lambda: pins.test_weight_gradient_linearity_identity(None)),
        ("golden_bn_act", lambda: [pins.test_golden_bn_act(None, l) for l in ("nhwc", "nchw")]),
        ("golden_multiplier", lambda: [pins.test_golden_multiplier(None, l) for l in ("nhwc", "nchw")]),
        ("torch_multiplier", lambda: pins.test_multiplier_gradients_equal_torch_autograd(None)),
        ("torch_multiplier_fwd", lambda: pins.test_multiplier_equals_torch_grouped_conv(None, False)),
        ("torch_bn_act", lambda: pins.test_bn_act_equals_torch_batch_norm_and_activations(None)),
    ]
    for name, fn in checks:
        try:
            fn()
        except Exception:  # noqa: BLE001 - any failure counts as detection
            failed.append(name)
    return failed


def _with_lib(path):
    lib = ctypes.CDLL(path)
    saved = oracle._lib
    oracle._lib = None
    real_build = oracle.build
    try:
        oracle._LIB_PATH_SAVED = oracle._LIB_PATH
        oracle._LIB_PATH = path
        oracle.build = lambda force=False: path
        oracle._load()
        return run_pin_subset()
    finally:
        oracle._LIB_PATH = oracle._LIB_PATH_SAVED
        oracle.build = real_build
        oracle._lib = saved
        del lib


def test_unmodified_oracle_passes_subset(tmp_path):
    assert _with_lib(build_variant(tmp_path, "original", None)) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    failed = _with_lib(build_variant(tmp_path, name, MUTANTS[name]))
    assert failed, f"planted mistake {name!r} went unnoticed by every pin"
