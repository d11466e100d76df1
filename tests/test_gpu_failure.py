"""The device-side failure path, exercised without faulting the GPU: a kernel
whose bounded mbarrier wait runs out (nothing ever arrives on the barrier)
raises the library's device error flag and returns; the host reads
GCONV_ERR_TIMEOUT through the C ABI, the flag clears on reading, and the CUDA
context keeps running correct convolutions afterwards."""
import ctypes

import numpy as np
import pytest
import torch

import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import build, inputs

from tolerance import assert_conv_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gc.library()


def test_bounded_wait_runs_out_and_reports_timeout(oracle_mod):
    lib = gc.library()
    assert lib.gconv_device_error_status() == gc.OK            # start from a clear flag
    s = torch.cuda.Stream()
    h = ctypes.c_void_p(s.cuda_stream)
    assert lib.gconv_selftest_wait_timeout(4096, h) == gc.OK
    assert lib.gconv_get_last_device_error(h) == gc.ERR_TIMEOUT
    assert lib.gconv_device_error_status() == gc.OK            # reading cleared it
    # the context is intact: a convolution on the same stream is still exact to the oracle
    d = inputs.conv_inputs(2, 32, 28, 28, 32, 3, 3, 32, seed=4600, x_dist="normal")
    with torch.cuda.stream(s):
        y = gc.conv2d(d["x"].cuda(), d["w"].cuda(), None, 1, 1, 1, 32)
    assert lib.gconv_get_last_device_error(h) == gc.OK
    ref, acc = oracle_mod.conv2d(d["x"], d["w"], None, 1, 1, 1, 32, return_absacc=True)
    assert_conv_close(y.cpu().numpy(), ref, acc, "conv after a timed-out wait")
    assert not np.isnan(y.cpu().numpy()).any()


def test_timeout_flag_is_per_device_state_not_sticky():
    """Two timeouts in a row each report once; valid work in between reports OK."""
    lib = gc.library()
    for _ in range(2):
        assert lib.gconv_selftest_wait_timeout(64, None) == gc.OK
        assert lib.gconv_get_last_device_error(None) == gc.ERR_TIMEOUT
        assert lib.gconv_get_last_device_error(None) == gc.OK
