"""The depthwise convolution inside a MobileNetV2 inverted-residual block
(x[4,24,56,56]: 1x1 24->144, BN, ReLU6, depthwise 3x3, BN, ReLU6, 1x1
144->24, residual add; "Fix the experiment" page), with the block's own
depthwise convolution replaced by this library's.

The substituted convolution is checked element by element against the FP64
oracle on the very input the block feeds it; the whole block output is then
checked against the same block computed on the CPU in float64 (oracle
depthwise convolution, float64 PyTorch CPU ops around it)."""
import numpy as np
import pytest
import torch

import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import block, build, inputs
from depthwise_convolution_fp32_b200 import workloads as wl

from tolerance import assert_conv_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gc.library()
    prm = inputs.mobilenet_block_inputs(wl.SEEDS["depthwise"] + 1)
    x = prm.pop("x")
    return x, prm


def test_substituted_depthwise_matches_oracle(setup, oracle_mod):
    x, prm = setup
    dev = block.to_device(prm, "cuda")
    prev = torch.backends.cudnn.allow_tf32
    torch.backends.cudnn.allow_tf32 = False
    try:
        h = block.expand(x.cuda(), dev)                  # the depthwise convolution's input
        d = block.library_depthwise(h, dev["wd"])
        torch.cuda.synchronize()
    finally:
        torch.backends.cudnn.allow_tf32 = prev
    assert gc.plan_name(4, 144, 56, 56, 144, 3, 3, 1, 1, 1, 144).startswith("direct")
    ref, absacc = oracle_mod.conv2d(h.cpu().numpy(), prm["wd"].numpy(), None, 1, 1, 1, 144, return_absacc=True)
    assert_conv_close(d.cpu().numpy(), ref, absacc, "block depthwise")


def test_block_output_matches_float64_block(setup, oracle_mod):
    x, prm = setup
    dev = block.to_device(prm, "cuda")
    prev = torch.backends.cudnn.allow_tf32
    torch.backends.cudnn.allow_tf32 = False
    try:
        y = block.forward(x.cuda(), dev, block.library_depthwise).cpu().double()
        h_gpu = block.expand(x.cuda(), dev).cpu()
    finally:
        torch.backends.cudnn.allow_tf32 = prev
    p64 = {k: ({kk: vv.double() for kk, vv in v.items()} if isinstance(v, dict) else v.double())
           for k, v in prm.items()}
    x64 = x.double()
    h64 = block.expand(x64, p64)
    # the FP32 GPU expansion differs from the float64 one by rounding only
    assert torch.allclose(h_gpu.double(), h64, rtol=1e-5, atol=1e-5)
    d64 = torch.from_numpy(oracle_mod.conv2d(h64.numpy(), prm["wd"].double().numpy(), None, 1, 1, 1, 144))
    y64 = block.project(x64, d64, p64)
    err = (y - y64).abs()
    # FP32 rounding through two BatchNorms, a ReLU6 and a 144-term 1x1 sum
    assert float((err / (1e-4 * (1.0 + y64.abs()))).max()) <= 1.0, float(err.max())


def test_fused_block_matches_float64_block(setup, oracle_mod):
    # depthwise conv + BatchNorm + ReLU6 in one call (conv2d_affine_clamp with the folded BatchNorm)
    x, prm = setup
    dev = block.to_device(prm, "cuda")
    prev = torch.backends.cudnn.allow_tf32
    torch.backends.cudnn.allow_tf32 = False
    try:
        y = block.forward_fused(x.cuda(), dev).cpu().double()
    finally:
        torch.backends.cudnn.allow_tf32 = prev
    p64 = {k: ({kk: vv.double() for kk, vv in v.items()} if isinstance(v, dict) else v.double())
           for k, v in prm.items()}
    x64 = x.double()
    d64 = torch.from_numpy(oracle_mod.conv2d(block.expand(x64, p64).numpy(), prm["wd"].double().numpy(),
                                             None, 1, 1, 1, 144))
    y64 = block.project(x64, d64, p64)
    err = (y - y64).abs()
    assert float((err / (1e-4 * (1.0 + y64.abs()))).max()) <= 1.0, float(err.max())
