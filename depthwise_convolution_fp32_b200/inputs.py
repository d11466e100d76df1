"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws random numbers; it holds none of the convolution or
GroupNorm arithmetic.  Every tensor is FP32, contiguous, on the CPU, drawn
from a ``torch.Generator`` seeded per workload, so the CUDA path and the CPU
oracle see bit-identical inputs.

Distributions follow the workloads the pages measure (the "GroupConv Atlas"
page: FP32 NCHW grouped 3x3 shapes; the POPCORNBENCH "Kimi-K2.6__l2_p21"
transcript: x[128,8,256,256], conv 8->32 3x3, bias/scale [32,1,1], GroupNorm
with 8 groups; the POPCORNBENCH "Kimi-K2.6__l1_p62" transcript:
x[8,32,512,512], conv 32->64 with a 5x9 kernel).
"""
from __future__ import annotations

import math

import torch


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def uniform(shape, lo, hi, g):
    return torch.rand(shape, generator=g, dtype=torch.float32).mul_(hi - lo).add_(lo)


def normal(shape, std, g, mean=0.0):
    return torch.randn(shape, generator=g, dtype=torch.float32).mul_(std).add_(mean)


def conv_inputs(N, C, H, W, K, R, S, groups, seed, x_dist="normal", w_bound=None,
                bias=False):
    """x[N,C,H,W] and w[K,C/groups,R,S] (and optionally bias[K]).

    x_dist: "normal" -> N(0,1); "uniform01" -> U[0,1); "uniform11" -> U[-1,1).
    w ~ U(-b, b) with b = w_bound or 1/sqrt(C/groups*R*S) (the default Conv2d
    initialisation bound); bias ~ U(-b, b) likewise."""
    g = generator(seed)
    if x_dist == "normal":
        x = normal((N, C, H, W), 1.0, g)
    elif x_dist == "uniform01":
        x = uniform((N, C, H, W), 0.0, 1.0, g)
    elif x_dist == "uniform11":
        x = uniform((N, C, H, W), -1.0, 1.0, g)
    else:
        raise ValueError(x_dist)
    cpg = C // groups
    b = w_bound if w_bound is not None else 1.0 / math.sqrt(cpg * R * S)
    w = uniform((K, cpg, R, S), -b, b, g)
    out = {"x": x, "w": w}
    if bias:
        out["bias"] = uniform((K,), -b, b, g)
    return out


def chain_inputs(N, C, H, W, K, R, S, groups, gn_groups, seed, bias_scale_std=0.02,
                 affine="identity"):
    """Inputs of the conv -> +bias -> *scale -> sigmoid -> GroupNorm chain.

    x ~ U[0,1); conv weight and conv bias ~ U(+-1/sqrt(fan_in)); the extra bias
    and the scale ~ N(0, bias_scale_std); GroupNorm gamma = 1, beta = 0 when
    affine == "identity", else gamma ~ U[0.5,1.5), beta ~ N(0, 0.5)."""
    g = generator(seed)
    x = uniform((N, C, H, W), 0.0, 1.0, g)
    cpg = C // groups
    bound = 1.0 / math.sqrt(cpg * R * S)
    w = uniform((K, cpg, R, S), -bound, bound, g)
    b_conv = uniform((K,), -bound, bound, g)
    b_extra = normal((K,), bias_scale_std, g)
    scale = normal((K,), bias_scale_std, g)
    if affine == "identity":
        gamma = torch.ones(K, dtype=torch.float32)
        beta = torch.zeros(K, dtype=torch.float32)
    else:
        gamma = uniform((K,), 0.5, 1.5, g)
        beta = normal((K,), 0.5, g)
    return {"x": x, "w": w, "b_conv": b_conv, "b_extra": b_extra, "scale": scale,
            "gamma": gamma, "beta": beta, "gn_groups": gn_groups}


def mobilenet_block_inputs(seed, N=4, cin=24, cexp=144, H=56, W=56):
    """Random-init parameters and input of one MobileNetV2 inverted-residual
    block (expansion 6: 1x1 conv cin->cexp, BN, ReLU6, depthwise 3x3, BN,
    ReLU6, 1x1 conv cexp->cin, residual add), the block the "Fix the
    experiment" page substitutes one convolution in.

    x ~ N(0,1); conv weights ~ U(+-1/sqrt(fan_in)); each BatchNorm (inference
    form) has gamma ~ U[0.5,1.5), beta ~ N(0,0.1), running mean ~ N(0,0.1),
    running var ~ U[0.5,1.5)."""
    g = generator(seed)
    x = normal((N, cin, H, W), 1.0, g)
    w1 = uniform((cexp, cin, 1, 1), -1.0 / math.sqrt(cin), 1.0 / math.sqrt(cin), g)
    wd = uniform((cexp, 1, 3, 3), -1.0 / 3.0, 1.0 / 3.0, g)
    w3 = uniform((cin, cexp, 1, 1), -1.0 / math.sqrt(cexp), 1.0 / math.sqrt(cexp), g)

    def bn(c):
        return {"gamma": uniform((c,), 0.5, 1.5, g), "beta": normal((c,), 0.1, g),
                "mean": normal((c,), 0.1, g), "var": uniform((c,), 0.5, 1.5, g)}
    return {"x": x, "w1": w1, "bn1": bn(cexp), "wd": wd, "bn2": bn(cexp), "w3": w3}
