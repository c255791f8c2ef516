"""Seeded synthetic workloads: the benchmark shapes of the source pages.

Shapes come from the llama.cpp PR "metal : add CONV_2D_DW" performance tables
(ggml shapes [W,H,C,N]: WHCN = NCHW, CWHN = NHWC) and its ASR encoder cases,
and from the MobileNet / Conformer / large-bandwidth configurations built on
them.  This module only draws random numbers: it holds none of the
convolution's arithmetic.  Output extents (needed for dy) are passed in by the
caller, who computes them with the library or the oracle.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)``
in the order x, W, b, dy, so the GPU path and the oracle read identical bytes.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple, Union

import torch


@dataclasses.dataclass(frozen=True)
class Case:
    name: str
    N: int
    H: int
    W: int
    C: int
    kH: int
    kW: int
    stride: Union[int, Tuple[int, int]] = 1
    dilation: Union[int, Tuple[int, int]] = 1
    padding: Union[str, int, Tuple[int, ...]] = "same"
    layout: str = "nhwc"
    wtype: str = "f32"
    act: str = "uniform"      # x and dy: "uniform" U(-1,1) or "normal" N(0,1)
    bias: bool = True         # b ~ U(-0.1, 0.1)
    seed: int = 0
    multiplier: int = 1       # output channels per input channel (C*multiplier outputs)

    def in_shape(self) -> Tuple[int, int, int, int]:
        if self.layout == "nhwc":
            return (self.N, self.H, self.W, self.C)
        return (self.N, self.C, self.H, self.W)

    @property
    def Co(self) -> int:
        return self.C * self.multiplier

    def out_shape(self, Ho: int, Wo: int) -> Tuple[int, int, int, int]:
        if self.layout == "nhwc":
            return (self.N, Ho, Wo, self.Co)
        return (self.N, self.Co, Ho, Wo)

    def with_(self, **kw) -> "Case":
        return dataclasses.replace(self, **kw)


def _act(gen: torch.Generator, shape, kind: str) -> torch.Tensor:
    if kind == "uniform":
        return torch.rand(shape, generator=gen, dtype=torch.float32) * 2.0 - 1.0
    if kind == "normal":
        return torch.randn(shape, generator=gen, dtype=torch.float32)
    raise ValueError(kind)


def make_inputs(case: Case, out_hw: Tuple[int, int]) -> Dict[str, Optional[torch.Tensor]]:
    """CPU float32 tensors x, w ([C*M,kH,kW], float32 or float16), b [C*M], dy.

    W ~ N(0, 1/(kH*kW)) (variance 1/(kH*kW)); with wtype "f16" the draw is
    rounded to float16 (round to nearest even), so `w` holds float16-exact
    values, and `w32` the same values in float32.
    """
    gen = torch.Generator().manual_seed(case.seed)
    x = _act(gen, case.in_shape(), case.act)
    w = torch.randn((case.Co, case.kH, case.kW), generator=gen, dtype=torch.float32)
    w = w * (1.0 / (case.kH * case.kW)) ** 0.5
    b = (torch.rand((case.Co,), generator=gen, dtype=torch.float32) * 0.2 - 0.1) if case.bias else None
    dy = _act(gen, case.out_shape(*out_hw), case.act)
    if case.wtype == "f16":
        w16 = w.to(torch.float16)
        return {"x": x, "w": w16, "w32": w16.to(torch.float32), "b": b, "dy": dy}
    return {"x": x, "w": w, "w32": w, "b": b, "dy": dy}


def make_bn(C: int, seed: int, eps: float = 1e-5) -> Tuple[torch.Tensor, torch.Tensor,
                                                          torch.Tensor, torch.Tensor, float]:
    """Inference-mode batch-norm statistics for the fused epilogue (CPU float32):
    gamma ~ U(0.25, 1.75), beta ~ U(-0.5, 0.5), running mean ~ U(-0.2, 0.2),
    running var ~ U(0.25, 2), drawn in that order from their own seed."""
    gen = torch.Generator().manual_seed(seed)
    u = lambda lo, hi: torch.rand((C,), generator=gen, dtype=torch.float32) * (hi - lo) + lo
    gamma = u(0.25, 1.75)
    beta = u(-0.5, 0.5)
    mean = u(-0.2, 0.2)
    var = u(0.25, 2.0)
    return gamma, beta, mean, var, eps


# ------------------------------------------------------------ configurations

def tiny() -> List[Case]:
    return [Case("tiny", 1, 8, 8, 4, 3, 3, padding="same", seed=1000)]


def mobilenet() -> List[Case]:
    """MobileNet-style NHWC f32; the stride-2 case uses explicit pad 1 on every
    side (the even-position decimation of stride-1 SAME, Ho = 28)."""
    return [
        Case("mobilenet_112x112x32_3x3", 1, 112, 112, 32, 3, 3, seed=1100),
        Case("mobilenet_56x56x128_5x5", 1, 56, 56, 128, 5, 5, seed=1101),
        Case("mobilenet_32x56x56x144_3x3_s2", 32, 56, 56, 144, 3, 3, stride=2, padding=1,
             seed=1102),
    ]


def conformer() -> List[Case]:
    out = []
    seed = 1200
    for layout in ("nhwc", "nchw"):
        for C, k in ((128, 15), (256, 31), (128, 31), (256, 15)):
            out.append(Case(f"conformer_1x24x{C}_1x{k}_{layout}", 1, 1, 24, C, 1, k,
                            layout=layout, act="normal", seed=seed))
            seed += 1
        out.append(Case(f"conformer_16x512x512_1x31_{layout}", 16, 1, 512, 512, 1, 31,
                        layout=layout, act="normal", seed=seed))
        seed += 1
    return out


def large() -> List[Case]:
    out = []
    seed = 1300
    for layout in ("nhwc", "nchw"):
        out.append(Case(f"large_512x512x256_3x3_{layout}", 1, 512, 512, 256, 3, 3,
                        layout=layout, seed=seed))
        seed += 1
        out.append(Case(f"large_30x19x128_7x7_{layout}", 1, 30, 19, 128, 7, 7,
                        layout=layout, seed=seed))
        seed += 1
    return out


def multiplier() -> List[Case]:
    """Channel multiplier: the grouped-gradient page's case (a 3x3 conv from 4
    to 8 channels, groups = 4, on a 4x4 input; W,H,C,N = 4,4,4,1) and a
    bandwidth-sized one, 1x512x512x128 -> 256 channels 3x3 SAME (the same
    output bytes as the large case), NHWC and NCHW."""
    out = [Case("mult_page_1x4x4x4_m2", 1, 4, 4, 4, 3, 3, padding=0, multiplier=2,
                act="uniform", seed=1500)]
    for i, layout in enumerate(("nhwc", "nchw")):
        out.append(Case(f"mult_512x512x128_m2_{layout}", 1, 512, 512, 128, 3, 3, layout=layout,
                        multiplier=2, seed=1501 + i))
    return out


def edge() -> List[Case]:
    """Mixed and edge cases: f16 weights, prime C, dilation 2/3, W = 1, N = 8,
    3x3/5x5/7x7, stride 2."""
    cases = []
    seed = 1400
    specs = [
        # (N, H, W, C, k, stride, dilation, padding, layout)
        (1, 13, 17, 7, 3, 1, 1, "same", "nhwc"),
        (2, 11, 9, 131, 3, 1, 1, "same", "nhwc"),
        (2, 11, 9, 131, 5, 2, 1, "same", "nchw"),
        (8, 9, 12, 16, 3, 1, 2, "same", "nhwc"),
        (8, 9, 12, 16, 3, 1, 3, "same", "nchw"),
        (1, 15, 16, 12, 5, 1, 2, (2, 3, 4, 1), "nhwc"),
        (3, 10, 1, 8, 3, 1, 1, "same", "nhwc"),
        (3, 10, 1, 8, 3, 1, 1, "same", "nchw"),
        (2, 1, 1, 5, 3, 1, 1, "same", "nhwc"),
        (8, 14, 14, 32, 7, 1, 1, "same", "nhwc"),
        (8, 14, 14, 32, 7, 2, 1, "same", "nchw"),
        (4, 15, 13, 24, 3, 2, 1, 1, "nhwc"),
        (4, 16, 16, 24, 3, 2, 1, "same", "nhwc"),
        (4, 16, 20, 8, 3, 2, 2, "same", "nhwc"),
        (2, 16, 20, 40, 5, 1, 1, "same", "nchw"),
        (2, 7, 64, 33, 1, 1, 1, "same", "nchw"),
    ]
    for (N, H, W, C, k, s, d, pad, layout) in specs:
        for wtype in ("f32", "f16"):
            name = f"edge_{N}x{H}x{W}x{C}_{k}x{k}_s{s}_d{d}_{layout}_{wtype}"
            cases.append(Case(name, N, H, W, C, k, k, stride=s, dilation=d, padding=pad,
                              layout=layout, wtype=wtype, seed=seed))
        seed += 1
    return cases


ALL = {"tiny": tiny, "mobilenet": mobilenet, "conformer": conformer, "large": large,
       "edge": edge}
