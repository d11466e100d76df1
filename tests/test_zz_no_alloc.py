"""The allocation-free fused chain, called through the C ABI.

Callers that cannot allocate device memory while they run (a CUDA graph being
recorded, an engine with a fixed memory budget, a host whose allocator belongs
to another framework) use gconv2d_bias_scale_sigmoid_groupnorm_fwd_noalloc,
which keeps its GroupNorm partial statistics in a fixed scratch array instead
of a cudaMalloc'd workspace.  These tests check, on two calls in a row (the
second call must not see anything the first left in the shared scratch), that
it returns what the regular entry point returns and that both agree with the
FP64 oracle within the chain's error bound, and that shapes needing more
scratch than the array holds are refused without launching.

This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import build, inputs

from tolerance import assert_chain_close, chain_tols

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    lib = gc.library()
    i, p, f = ctypes.c_int, ctypes.c_void_p, ctypes.c_float
    fn = lib.gconv2d_bias_scale_sigmoid_groupnorm_fwd_noalloc
    fn.restype = i
    fn.argtypes = [p, p, p] + [i] * 11 + [p, i, p, p, f, p, p]
    lib.gconv_noalloc_scratch_capacity.restype = ctypes.c_size_t
    lib.gconv_noalloc_scratch_capacity.argtypes = []
    return lib


def _call(fn, dev, geo, gn, eps, out):
    N, C, H, W, K, R, S, st, pad, dil, g = geo
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(dev["x"].data_ptr(), dev["w"].data_ptr(), dev["bias"].data_ptr(), N, C, H, W, K, R, S,
              st, pad, dil, g, dev["scale"].data_ptr(), gn, dev["gamma"].data_ptr(),
              dev["beta"].data_ptr(), eps, out.data_ptr(), stream)


def _device_inputs(d):
    return {"x": d["x"].cuda(), "w": d["w"].cuda(), "bias": (d["b_conv"] + d["b_extra"]).cuda(),
            "scale": d["scale"].cuda(), "gamma": d["gamma"].cuda(), "beta": d["beta"].cuda()}


@pytest.mark.parametrize("geo,gn,std", [
    ((4, 8, 66, 70, 32, 3, 3, 1, 0, 1, 1), 8, 1.0),     # the fused-chain geometry, small
    ((2, 16, 30, 30, 16, 3, 3, 1, 1, 1, 16), 4, 0.5),   # depthwise conv in the chain
])
def test_noalloc_matches_regular_entry_point_twice(lib, oracle_mod, geo, gn, std):
    N, C, H, W, K, R, S, st, pad, dil, g = geo
    P, Q = gc.output_size(H, W, R, S, st, pad, dil)
    eps = 1e-5
    for call in range(2):        # two calls in a row on different inputs
        d = inputs.chain_inputs(N, C, H, W, K, R, S, g, gn, seed=900 + 17 * call,
                                bias_scale_std=std, affine="random")
        dev = _device_inputs(d)
        y_ref = torch.full((N, K, P, Q), float("nan"), device="cuda")
        y_new = torch.full((N, K, P, Q), float("nan"), device="cuda")
        assert _call(lib.gconv2d_bias_scale_sigmoid_groupnorm_fwd, dev, geo, gn, eps, y_ref) == gc.OK
        assert _call(lib.gconv2d_bias_scale_sigmoid_groupnorm_fwd_noalloc, dev, geo, gn, eps,
                     y_new) == gc.OK
        torch.cuda.synchronize()
        ref = oracle_mod.chain(d["x"], d["w"], d["b_conv"], d["b_extra"], d["scale"], gn,
                               d["gamma"], d["beta"], eps, st, pad, dil, g)
        _, tau_y = chain_tols(ref, d["scale"].numpy(), d["gamma"].numpy(), eps, K // gn)
        a = y_new.cpu().numpy().astype(np.float64)
        b = y_ref.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(a - b) <= tau_y), f"call {call}: max diff {np.nanmax(np.abs(a - b))}"
        # and each result against the oracle directly, so a fault both paths share cannot hide
        assert_chain_close(a, ref, d["scale"].numpy(), d["gamma"].numpy(), eps, K // gn, f"noalloc call {call}")
        assert_chain_close(b, ref, d["scale"].numpy(), d["gamma"].numpy(), eps, K // gn, f"regular call {call}")
    assert lib.gconv_device_error_status() == gc.OK


def test_noalloc_refuses_shapes_beyond_capacity(lib):
    # 16384 images x 32 GroupNorm groups of one channel: at least one 16-byte
    # partial per (image, group) is 8 MiB whatever the tiling, more than the
    # fixed scratch array (small 4x4 planes keep the buffers small)
    geo = (16384, 8, 4, 4, 32, 3, 3, 1, 0, 1, 1)
    gn = 32
    N, C, H, W, K, R, S, st, pad, dil, g = geo
    assert N * gn * 16 > lib.gconv_noalloc_scratch_capacity()
    P, Q = gc.output_size(H, W, R, S, st, pad, dil)
    # real, correctly sized buffers: nothing may be launched, but nothing
    # could go out of bounds if it were
    dev = {"x": torch.zeros(N, C, H, W, device="cuda"), "w": torch.zeros(K, C, R, S, device="cuda"),
           "bias": torch.zeros(K, device="cuda"), "scale": torch.ones(K, device="cuda"),
           "gamma": torch.ones(K, device="cuda"), "beta": torch.zeros(K, device="cuda")}
    y = torch.full((N, K, P, Q), 7.0, device="cuda")
    st_code = _call(lib.gconv2d_bias_scale_sigmoid_groupnorm_fwd_noalloc, dev, geo, gn, 1e-5, y)
    torch.cuda.synchronize()
    assert st_code == gc.ERR_WORKSPACE
    assert bool((y == 7.0).all()), "a refused call must not write the output"
