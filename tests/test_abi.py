"""The C ABI without a GPU: the library builds and loads, exports every entry
point include/gconv.h declares, and rejects invalid arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gc.library()


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"^GCONV_API\s[^;(]*?\b(\w+)\s*\(", src, re.M)
    return names


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "gconv2d_fwd" in names and "gconv2d_bias_scale_sigmoid_groupnorm_fwd" in names
    for n in names:
        assert hasattr(lib, n), n
    out = os.popen(f"nm -D --defined-only {gc.library_path()}").read()
    exported = set(re.findall(r" T (\w+)$", out, re.M))
    assert set(names) <= exported
    # nothing else leaks out of the library but the C ABI
    assert {e for e in exported if not e.startswith("_")} == set(names)


def test_status_strings(lib):
    for st in range(6):
        assert gc.status_string(st).startswith("GCONV_")
    assert "unknown" in gc.status_string(42)
    assert "sm_100a" in gc.version()


def test_output_size_matches_pages(lib, oracle_mod):
    assert gc.output_size(512, 512, 5, 9) == (508, 504)
    assert gc.output_size(256, 256, 3, 3) == (254, 254)
    assert gc.output_size(56, 56, 3, 3, 1, 1, 1) == (56, 56)
    for (H, R, st, p, d) in [(7, 3, 2, 1, 1), (9, 5, 1, 4, 2), (14, 3, 2, 0, 1), (1, 1, 1, 0, 1)]:
        assert gc.output_size(H, H, R, R, st, p, d)[0] == oracle_mod.out_extent(H, R, st, p, d)
    with pytest.raises(gc.GconvError) as e:
        gc.output_size(4, 4, 7, 7)
    assert e.value.status == gc.ERR_INVALID_ARG


FAKE = 0x10000  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("args", [
    dict(N=0), dict(C=0), dict(H=0), dict(K=0), dict(R=0), dict(stride=0), dict(pad=-1),
    dict(dilation=0), dict(groups=0), dict(groups=4), dict(C=8, groups=3), dict(R=11, S=11),
])
def test_conv_rejects_invalid_sizes(lib, args):
    a = dict(N=1, C=6, H=8, W=8, K=6, R=3, S=3, stride=1, pad=1, dilation=1, groups=2)
    a.update(args)
    st = lib.gconv2d_fwd(FAKE, FAKE, None, a["N"], a["C"], a["H"], a["W"], a["K"], a["R"], a["S"],
                         a["stride"], a["pad"], a["dilation"], a["groups"], FAKE, None)
    assert st == gc.ERR_INVALID_ARG


def test_conv_rejects_bad_pointers(lib):
    geo = (1, 4, 8, 8, 4, 3, 3, 1, 1, 1, 4)
    assert lib.gconv2d_fwd(None, FAKE, None, *geo, FAKE, None) == gc.ERR_INVALID_ARG
    assert lib.gconv2d_fwd(FAKE, None, None, *geo, FAKE, None) == gc.ERR_INVALID_ARG
    assert lib.gconv2d_fwd(FAKE, FAKE, None, *geo, None, None) == gc.ERR_INVALID_ARG
    assert lib.gconv2d_fwd(FAKE + 2, FAKE, None, *geo, FAKE, None) == gc.ERR_INVALID_ARG
    assert lib.gconv2d_fwd(FAKE, FAKE, FAKE + 1, *geo, FAKE, None) == gc.ERR_INVALID_ARG


def test_chain_rejects_invalid_arguments(lib):
    geo = (2, 8, 10, 10, 32, 3, 3, 1, 0, 1, 1)
    f = lib.gconv2d_bias_scale_sigmoid_groupnorm_fwd
    ok = dict(scale=FAKE, gn=8, gamma=FAKE, beta=FAKE, eps=1e-5)
    def call(**kw):
        d = dict(ok)
        d.update(kw)
        return f(FAKE, FAKE, None, *geo, d["scale"], d["gn"], d["gamma"], d["beta"], d["eps"], FAKE, None)
    assert call(gn=0) == gc.ERR_INVALID_ARG
    assert call(gn=5) == gc.ERR_INVALID_ARG
    assert call(scale=None) == gc.ERR_INVALID_ARG
    assert call(gamma=None) == gc.ERR_INVALID_ARG
    assert call(beta=None) == gc.ERR_INVALID_ARG
    assert call(eps=-1.0) == gc.ERR_INVALID_ARG
    assert call(eps=float("nan")) == gc.ERR_INVALID_ARG
    assert call(gamma=FAKE + 2) == gc.ERR_INVALID_ARG


def _table_family(shape, chain=0):
    """The family the compiled-in measured table picks for a shape, or None."""
    import json
    path = os.path.join(ROOT, "depthwise_convolution_fp32_b200", "dispatch_table.json")
    if not os.path.exists(path):
        return None
    for e in json.load(open(path))["entries"]:
        if e["shape"] == list(shape) and e.get("chain", 0) == chain:
            return e["best"].split(":")[0]
    return None


def test_plan_names(lib):
    # the headline depthwise workload: the measured table's choice, else (14 MB, latency-bound) blocked
    fam = _table_family((4, 144, 56, 56, 144, 3, 3, 1, 1, 1, 144))
    want = "direct_stream_3x3s1p1" if fam == "direct_stream" else "direct_tma_3x3s1p1"
    assert gc.plan_name(4, 144, 56, 56, 144, 3, 3, 1, 1, 1, 144) == want
    # outside the table: an 822 MB depthwise problem streams
    assert gc.plan_name(32, 256, 112, 112, 256, 3, 3, 1, 1, 1, 256, 0) in (
        "direct_stream_3x3s1p1" if _table_family((32, 256, 112, 112, 256, 3, 3, 1, 1, 1, 256)) in
        (None, "direct_stream") else "direct_tma_3x3s1p1",)
    assert gc.plan_name(2, 16, 14, 14, 16, 3, 3, 1, 1, 1, 16) == "direct_3x3s1p1"   # rows not 16-byte multiples
    assert gc.plan_name(16, 64, 128, 128, 64, 3, 3, 2, 1, 1, 64) == "direct_stream_3x3s2p1"
    # the fused chain's conv stage never streams (its epilogue reduces statistics per CTA)
    assert not gc.plan_name(2, 16, 30, 32, 16, 3, 3, 1, 1, 1, 16, chain=True).startswith("direct_stream")
    assert gc.plan_name(1, 8, 16, 16, 8, 3, 3, 1, 1, 2, 4) == "direct_generic"
    assert gc.plan_name(1, 8, 16, 16, 8, 3, 3, 1, 1, 1, 3) == "invalid"
    assert gc.chain_workspace_size(128, 8, 256, 256, 32, 3, 3, 1, 0, 1, 1, 8) > 0
    assert gc.chain_workspace_size(128, 8, 256, 256, 32, 3, 3, 1, 0, 1, 1, 5) == 0


def test_force_kernel_names(lib):
    for n in ("generic", "direct", "direct_cpasync", "direct_blocked", "direct_stream", "igemm", "igemm_split",
              "igemm_fused", "winograd", "direct_stream:kt2", "direct_blocked:kt8", "auto"):
        gc.force_kernel(n)
    gc.force_kernel("direct_blocked")
    try:
        assert gc.plan_name(4, 144, 56, 56, 144, 3, 3, 1, 1, 1, 144) == "direct_tma_3x3s1p1"
    finally:
        gc.force_kernel("auto")
    for bad in ("cudnn", "igemm:kt4", "auto:kt2", "direct:kt3", "direct_stream:", "winograd:kt4"):
        with pytest.raises(gc.GconvError):
            gc.force_kernel(bad)
    gc.force_kernel("auto")


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 8, 8)
    w = torch.zeros(4, 1, 3, 3)
    with pytest.raises(ValueError):
        gc.conv2d(x, w, padding=1, groups=4)


def test_affine_clamp_rejects_bad_bounds(lib):
    geo = (1, 4, 8, 8, 4, 3, 3, 1, 1, 1, 4)
    f = lib.gconv2d_affine_clamp_fwd
    assert f(FAKE, FAKE, *geo, None, None, 1.0, 0.0, FAKE, None) == gc.ERR_INVALID_ARG
    assert f(FAKE, FAKE, *geo, None, None, float("nan"), 1.0, FAKE, None) == gc.ERR_INVALID_ARG


def test_selftest_wait_timeout_rejects_bad_limits(lib):
    # validated on the host: nothing is launched
    assert lib.gconv_selftest_wait_timeout(0, None) == gc.ERR_INVALID_ARG
    assert lib.gconv_selftest_wait_timeout((1 << 24) + 1, None) == gc.ERR_INVALID_ARG


def test_per_axis_entry_point_validates_and_plans(lib):
    f = lib.gconv2d_fwd_ex
    geo = (1, 4, 8, 8, 4, 3, 3)
    # each per-axis value checked on its own
    for bad in [(0, 1, 1, 1, 1, 1), (1, 0, 1, 1, 1, 1), (1, 1, -1, 1, 1, 1), (1, 1, 1, -1, 1, 1),
                (1, 1, 1, 1, 0, 1), (1, 1, 1, 1, 1, 0), (1, 1, 0, 0, 5, 1)]:
        assert f(FAKE, FAKE, None, *geo, *bad, 4, FAKE, None) == gc.ERR_INVALID_ARG, bad
    # unequal axes use the general-geometry kernel; equal axes plan like gconv2d_fwd
    assert gc.plan_name(2, 16, 30, 34, 16, 3, 3, (1, 2), (1, 0), 1, 16) == "direct_generic"
    assert gc.plan_name(2, 32, 24, 36, 64, 5, 9, 1, (2, 4), 1, 1).startswith("igemm_tf32_bf16x")
    assert gc.plan_name(4, 144, 56, 56, 144, 3, 3, (1, 1), (1, 1), (1, 1), 144) == \
        gc.plan_name(4, 144, 56, 56, 144, 3, 3, 1, 1, 1, 144)


def test_peaks_library_exports_its_microbenchmarks():
    """The benchmark's roofline microbenchmarks build as their own library
    (not part of the C ABI) and export their three entry points."""
    lib = ctypes.CDLL(build.build_peaks())
    for name in ("gpeaks_ffma", "gpeaks_mma_tf32", "gpeaks_mma_bf16"):
        assert hasattr(lib, name), name
