"""Run one named workload for a few calls, optionally at a reduced batch, as a
target for a profiler (ncu captures of one kernel on a small case).

    python -m depthwise_convolution_fp32_b200.profile_case --workload dense_5x9 --batch 2 --calls 2

Inputs are the seeded synthetic ones of the workload; only the library's own
CUDA path runs (one call per --calls, each followed by a synchronize).
"""
from __future__ import annotations

import argparse
import dataclasses

import torch

import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import inputs
from depthwise_convolution_fp32_b200 import workloads as wl


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="depthwise",
                    choices=["tiny_grouped", "depthwise", "dense_5x9", "fused_chain"])
    ap.add_argument("--batch", type=int, default=0, help="override N (0: the workload's own)")
    ap.add_argument("--calls", type=int, default=2)
    args = ap.parse_args()
    if not torch.cuda.is_available():
        raise SystemExit("a CUDA device is required")
    seed = wl.SEEDS[args.workload]
    if args.workload == "fused_chain":
        ch = wl.FUSED_CHAIN   # eps 1e-5
        s = ch.conv if args.batch <= 0 else dataclasses.replace(ch.conv, N=args.batch)
        d = inputs.chain_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.groups, ch.gn_groups, seed)
        x, w = d["x"].cuda(), d["w"].cuda()
        b = (d["b_conv"] + d["b_extra"]).cuda()
        sc, ga, be = d["scale"].cuda(), d["gamma"].cuda(), d["beta"].cuda()

        def run():
            return gc.conv2d_bias_scale_sigmoid_groupnorm(x, w, b, sc, ch.gn_groups, ga, be, 1e-5,
                                                          s.stride, s.pad, s.dil, s.groups)
    else:
        s0 = {"tiny_grouped": wl.TINY_GROUPED, "depthwise": wl.DEPTHWISE, "dense_5x9": wl.DENSE_5X9}[args.workload]
        s = s0 if args.batch <= 0 else dataclasses.replace(s0, N=args.batch)
        x_dist = "uniform01" if args.workload == "dense_5x9" else "normal"
        d = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.groups, seed, x_dist=x_dist)
        x, w = d["x"].cuda(), d["w"].cuda()

        def run():
            return gc.conv2d(x, w, None, s.stride, s.pad, s.dil, s.groups)
    for _ in range(args.calls):
        y = run()
        torch.cuda.synchronize()
    plan = gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups,
                        chain=args.workload == "fused_chain")
    print(f"{args.workload} N={s.N} plan={plan} y={tuple(y.shape)} mean|y|={float(y.abs().mean()):.6f}")


if __name__ == "__main__":
    main()
