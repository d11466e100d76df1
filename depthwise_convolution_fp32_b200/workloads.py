"""Workload definitions: the shapes the pages measure, and the algorithmic work
(bytes that must cross HBM, multiply-accumulates) of each.

Shapes:
  tiny_grouped  x[1,8,16,16], w[8,2,3,3], groups=4, 3x3 s1 p1      (parity case)
  depthwise     x[4,144,56,56], w[144,1,3,3], groups=144, 3x3 s1 p1
                (the depthwise conv of a MobileNetV2 inverted-residual block;
                 "GroupConv Atlas", MobileNetV2 features[3] module probe)
  sweep80       80 grouped 3x3 s1 p1 shapes, K=C, channels/group in {1,2,4,8}
                ("GroupConv Atlas", "Fix the experiment"; the page's own shape
                 list is unpublished, so a seeded permutation stands in for it)
  fused_chain   x[128,8,256,256], conv 8->32 3x3 p0, +bias, *scale, sigmoid,
                GroupNorm(8 groups)  (POPCORNBENCH Kimi-K2.6__l2_p21 Model)
  dense_5x9     x[8,32,512,512], w[64,32,5,9], p0 -> y[8,64,508,504]
                (POPCORNBENCH Kimi-K2.6__l1_p62 problem statement)
"""
from __future__ import annotations

import dataclasses
import itertools
import math

import numpy as np

F32 = 4  # bytes per element


@dataclasses.dataclass(frozen=True)
class ConvShape:
    N: int
    C: int
    H: int
    W: int
    K: int
    R: int
    S: int
    stride: int = 1
    pad: int = 0
    dil: int = 1
    groups: int = 1
    bias: bool = False

    @property
    def P(self) -> int:
        return (self.H + 2 * self.pad - self.dil * (self.R - 1) - 1) // self.stride + 1

    @property
    def Q(self) -> int:
        return (self.W + 2 * self.pad - self.dil * (self.S - 1) - 1) // self.stride + 1

    @property
    def cpg(self) -> int:
        return self.C // self.groups

    @property
    def n_out(self) -> int:
        return self.N * self.K * self.P * self.Q

    @property
    def macs(self) -> int:
        """Multiply-accumulates of the dense definition (every tap, padding
        taps included, as a GEMM view counts them)."""
        return self.n_out * self.cpg * self.R * self.S

    @property
    def flops(self) -> int:
        return 2 * self.macs

    @property
    def bytes(self) -> int:
        """Algorithmic HBM bytes: x read once, w read once, y written once."""
        b = (self.N * self.C * self.H * self.W + self.K * self.cpg * self.R * self.S
             + self.n_out) * F32
        if self.bias:
            b += self.K * F32
        return b

    def label(self) -> str:
        return (f"x[{self.N},{self.C},{self.H},{self.W}] w[{self.K},{self.cpg},{self.R},{self.S}]"
                f" g={self.groups} s{self.stride} p{self.pad} d{self.dil}")


@dataclasses.dataclass(frozen=True)
class ChainShape:
    conv: ConvShape
    gn_groups: int

    @property
    def bytes(self) -> int:
        """x once, w + conv bias + extra bias + scale + gamma + beta, y once."""
        c = self.conv
        return (c.N * c.C * c.H * c.W + c.K * c.cpg * c.R * c.S + 5 * c.K + c.n_out) * F32

    @property
    def flops(self) -> int:
        return self.conv.flops


TINY_GROUPED = ConvShape(N=1, C=8, H=16, W=16, K=8, R=3, S=3, stride=1, pad=1, groups=4)
DEPTHWISE = ConvShape(N=4, C=144, H=56, W=56, K=144, R=3, S=3, stride=1, pad=1, groups=144)
FUSED_CHAIN = ChainShape(ConvShape(N=128, C=8, H=256, W=256, K=32, R=3, S=3, stride=1, pad=0,
                                   groups=1, bias=True), gn_groups=8)
DENSE_5X9 = ConvShape(N=8, C=32, H=512, W=512, K=64, R=5, S=9, stride=1, pad=0, groups=1)


def sweep80() -> list[ConvShape]:
    """The 80-shape grouped sweep: the 320-tuple cross product
    N x C x channels-per-group x H (nested in that order) permuted with
    numpy.random.default_rng(0), first 80 kept; 3x3, s1, p1, d1, K=C."""
    tuples = list(itertools.product((1, 4, 16, 32), (32, 64, 128, 256, 512),
                                    (1, 2, 4, 8), (14, 28, 56, 112)))
    order = np.random.default_rng(0).permutation(len(tuples))[:80]
    out = []
    for i in order:
        N, C, cpg, H = tuples[int(i)]
        out.append(ConvShape(N=N, C=C, H=H, W=H, K=C, R=3, S=3, stride=1, pad=1,
                             groups=C // cpg))
    return out


def sweep_seed(i: int) -> int:
    return 3000 + i


SEEDS = {"tiny_grouped": 1001, "depthwise": 1002, "fused_chain": 1004, "dense_5x9": 1005}

# Shapes around the implicit-GEMM threshold (channels per group x taps near
# 64, output channels per group at the tensor path's minimum of 32), timed for
# the dispatch table: (N, C, H, W, K, R = S, pad, groups); seeds 5000 + index.
THRESHOLD_RING = [
    (8, 32, 56, 56, 32, 3, 1, 1), (8, 64, 56, 56, 64, 3, 1, 1), (8, 128, 28, 28, 128, 3, 1, 4),
    (8, 16, 56, 56, 32, 3, 1, 1), (8, 8, 128, 128, 32, 3, 1, 1), (8, 64, 56, 56, 64, 1, 0, 1),
    (8, 128, 28, 28, 128, 1, 0, 1), (8, 256, 28, 28, 256, 3, 1, 8),
]


def roofline_time_s(shape: ConvShape, hbm_gbs: float, fp32_tflops: float) -> tuple[float, str]:
    """max(bytes / HBM bandwidth, FLOPs / FP32 peak) and the binding term."""
    tb = shape.bytes / (hbm_gbs * 1e9)
    tf = shape.flops / (fp32_tflops * 1e12)
    return (tb, "hbm") if tb >= tf else (tf, "fp32")


def fp32_fma_peak_tflops(sm_count: int = 148, clock_mhz: float = 1965.0) -> float:
    """CUDA-core FP32 peak: 128 FMA lanes per SM, 2 FLOP per FMA."""
    return sm_count * 128 * 2 * clock_mhz * 1e6 / 1e12


assert math.isclose(fp32_fma_peak_tflops(), 74.44, rel_tol=1e-3)
