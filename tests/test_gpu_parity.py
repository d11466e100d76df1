"""GPU parity: every kernel path against the FP64 oracle on the same seeded
inputs, element by element, through the C ABI (via the ctypes binding).

Small and medium shapes are compared in full; the full-size workloads are
compared on sampled outputs the oracle computes one by one (and whole
GroupNorm groups for the chain).  Output buffers are NaN-prefilled and
surrounded by canary guards, so a missed store or a stray one fails."""
import ctypes
import math
import zlib

import numpy as np
import pytest
import torch

import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import build, inputs
from depthwise_convolution_fp32_b200 import workloads as wl

from tolerance import assert_chain_close, assert_conv_close

pytestmark = pytest.mark.gpu

CANARY = 1234.5678


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gc.library()
    gc.force_kernel("auto")
    yield
    gc.force_kernel("auto")


class Guarded:
    """A NaN-prefilled output with canary regions on both sides; `misalign`
    shifts the output start by that many floats (4-byte aligned only)."""

    def __init__(self, shape, guard=1024, misalign=0):
        self.n = int(np.prod(shape))
        self.g = guard + misalign
        self.buf = torch.full((self.n + 2 * guard + misalign,), CANARY, device="cuda")
        self.buf[self.g:self.g + self.n] = float("nan")
        self.y = self.buf[self.g:self.g + self.n].view(*shape)

    def check(self):
        lo = self.buf[:self.g]
        hi = self.buf[self.g + self.n:]
        assert bool((lo == CANARY).all()) and bool((hi == CANARY).all()), "write outside y"


def _to_dev(t, misalign=0):
    if misalign == 0:
        return t.cuda()
    buf = torch.empty(t.numel() + misalign, device="cuda")
    v = buf[misalign:misalign + t.numel()].view(t.shape)
    v.copy_(t)
    return v


def run_conv(d, stride, pad, dil, groups, misalign=0):
    x = _to_dev(d["x"], misalign)
    w = d["w"].cuda()
    b = d["bias"].cuda() if "bias" in d else None
    N, C, H, W = d["x"].shape
    K, _, R, S = d["w"].shape
    P, Q = gc.output_size(H, W, R, S, stride, pad, dil)
    out = Guarded((N, K, P, Q), misalign=misalign)
    gc.conv2d(x, w, b, stride, pad, dil, groups, out=out.y)
    torch.cuda.synchronize()
    out.check()
    return out.y


def full_check(oracle_mod, d, stride, pad, dil, groups, what, misalign=0):
    y = run_conv(d, stride, pad, dil, groups, misalign).cpu().numpy()
    ref, acc = oracle_mod.conv2d(d["x"], d["w"], d.get("bias"), stride, pad, dil, groups,
                                 return_absacc=True)
    return assert_conv_close(y, ref, acc, what)


def sampled_idx(shape, n_random, seed):
    """Random flat indices plus every border position of a few output planes."""
    N, K, P, Q = shape
    rng = np.random.default_rng(seed)
    idx = set(rng.integers(0, N * K * P * Q, n_random).tolist())
    for (n, k) in [(0, 0), (N - 1, K - 1), (N // 2, K // 2)]:
        base = (n * K + k) * P * Q
        for p in range(P):
            for q in (0, 1, Q - 2, Q - 1):
                if 0 <= q < Q:
                    idx.add(base + p * Q + q)
        for q in range(Q):
            for p in (0, P - 1):
                idx.add(base + p * Q + q)
    return np.array(sorted(idx), dtype=np.int64)


def sampled_check(oracle_mod, d, y_dev, stride, pad, dil, groups, what, n_random=4000, seed=0):
    idx = sampled_idx(tuple(y_dev.shape), n_random, seed)
    got = y_dev.reshape(-1)[torch.from_numpy(idx).cuda()].cpu().numpy()
    ref, acc = oracle_mod.conv2d_at(d["x"], d["w"], idx, d.get("bias"), stride, pad, dil, groups)
    return assert_conv_close(got, ref, acc, what)


# ------------------------------------------------------------------ workloads

@pytest.mark.parametrize("j", range(len(wl.THRESHOLD_RING)))
def test_threshold_ring_default_dispatch(oracle_mod, j):
    """The dispatch-table shapes around the implicit-GEMM threshold (several run
    on the tensor cores with folded tap rows) through the default dispatch."""
    N, C, H, W, K, R, pad, g = wl.THRESHOLD_RING[j]
    d = inputs.conv_inputs(N, C, H, W, K, R, R, g, 5000 + j, x_dist="normal",
                           w_bound=1 / math.sqrt(R * R * (C // g)))
    y = run_conv(d, 1, pad, 1, g)
    sampled_check(oracle_mod, d, y, 1, pad, 1, g, f"ring {j} {gc.plan_name(N, C, H, W, K, R, R, 1, pad, 1, g)}",
                  n_random=6000, seed=j)
    assert gc.library().gconv_device_error_status() == gc.OK


def test_tiny_grouped_full(oracle_mod):
    s = wl.TINY_GROUPED
    d = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.groups, wl.SEEDS["tiny_grouped"],
                           x_dist="uniform11", w_bound=1 / math.sqrt(18))
    full_check(oracle_mod, d, 1, 1, 1, s.groups, "tiny grouped")


def test_depthwise_mobilenet_full(oracle_mod):
    s = wl.DEPTHWISE
    d = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.groups, wl.SEEDS["depthwise"],
                           x_dist="normal", w_bound=1 / 3)
    full_check(oracle_mod, d, 1, 1, 1, s.groups, "depthwise 4x144x56x56")


@pytest.mark.parametrize("i", range(80))
def test_sweep80(oracle_mod, i):
    s = wl.sweep80()[i]
    d = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, 3, 3, s.groups, wl.sweep_seed(i),
                           x_dist="normal", w_bound=1 / math.sqrt(9 * s.cpg))
    if s.macs <= 4e8:
        full_check(oracle_mod, d, 1, 1, 1, s.groups, s.label())
    else:
        y = run_conv(d, 1, 1, 1, s.groups)
        sampled_check(oracle_mod, d, y, 1, 1, 1, s.groups, s.label(), seed=i)


def test_dense_5x9_full_size_sampled(oracle_mod):
    s = wl.DENSE_5X9
    d = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, 1, wl.SEEDS["dense_5x9"],
                           x_dist="uniform01", w_bound=1 / math.sqrt(1440))
    y = run_conv(d, 1, 0, 1, 1)
    assert tuple(y.shape) == (8, 64, 508, 504)
    sampled_check(oracle_mod, d, y, 1, 0, 1, 1, "dense 5x9 full size", n_random=3000)


def test_dense_5x9_small_full(oracle_mod):
    d = inputs.conv_inputs(1, 32, 37, 70, 64, 5, 9, 1, 77, x_dist="uniform01",
                           w_bound=1 / math.sqrt(1440))
    full_check(oracle_mod, d, 1, 0, 1, 1, "dense 5x9 ragged")


# ------------------------------------------------------------------ geometry

GEOMS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, bias
    (2, 16, 14, 14, 16, 3, 3, 1, 1, 1, 16, False),   # W=14: 4-byte staging path
    (1, 32, 28, 28, 32, 3, 3, 1, 1, 1, 8, True),
    (3, 12, 17, 23, 12, 3, 3, 1, 1, 1, 12, True),     # odd sizes, ragged tiles
    (2, 8, 33, 130, 8, 3, 3, 1, 1, 1, 8, False),     # Q > 128: two column tiles
    (1, 16, 56, 56, 32, 3, 3, 1, 1, 1, 16, False),   # channel multiplier 2
    (2, 24, 20, 20, 48, 3, 3, 1, 1, 1, 3, True),     # cpg 8, kpg 16
    (1, 8, 29, 31, 8, 3, 3, 2, 1, 1, 8, False),      # stride 2 depthwise
    (2, 16, 56, 56, 16, 3, 3, 2, 1, 1, 16, True),
    (1, 8, 19, 21, 16, 3, 3, 1, 0, 1, 1, True),      # pad 0 dense
    (1, 16, 12, 40, 16, 1, 1, 1, 0, 1, 4, True),     # pointwise grouped
    (1, 8, 15, 15, 8, 3, 3, 1, 2, 2, 8, False),      # dilation 2 (generic)
    (2, 6, 11, 13, 9, 5, 3, 1, 2, 1, 3, True),       # R != S (generic)
    (1, 4, 9, 9, 8, 7, 7, 1, 3, 1, 2, False),        # 7x7 (generic)
    (1, 6, 10, 12, 6, 3, 3, 3, 1, 1, 6, False),      # stride 3 (generic)
    (1, 4, 1, 17, 4, 1, 3, 1, 0, 1, 4, False),       # H = 1
    (1, 4, 5, 1, 4, 3, 1, 1, 1, 1, 2, False),        # W = 1
    (1, 3, 3, 3, 5, 3, 3, 1, 0, 1, 1, True),         # P = Q = 1
    (1, 8, 6, 6, 8, 3, 3, 1, 4, 1, 8, False),        # padding larger than the halo chunk
    (1, 64, 9, 9, 64, 3, 3, 1, 1, 1, 1, False),      # dense 3x3, cpg 64 (channel chunks)
    (1, 96, 7, 12, 12, 5, 9, 1, 0, 1, 1, False),     # dense 5x9 with many channels
]


@pytest.mark.parametrize("geo", GEOMS, ids=lambda g: "x".join(map(str, g[:11])))
def test_geometry_full(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=zlib.crc32(repr(geo).encode()) % 10000, x_dist="normal",
                           bias=bias)
    full_check(oracle_mod, d, st, pad, dil, g, str(geo))


@pytest.mark.parametrize("geo", GEOMS[:10], ids=lambda g: "x".join(map(str, g[:11])))
def test_forced_generic_matches_oracle(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=7 + zlib.crc32(repr(geo).encode()) % 1000, x_dist="normal",
                           bias=bias)
    gc.force_kernel("generic")
    try:
        full_check(oracle_mod, d, st, pad, dil, g, "generic " + str(geo))
    finally:
        gc.force_kernel("auto")


@pytest.mark.parametrize("geo", GEOMS[:10], ids=lambda g: "x".join(map(str, g[:11])))
def test_forced_cpasync_staging_matches_oracle(oracle_mod, geo):
    """The cp.async staging path on shapes that would otherwise use TMA."""
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=11 + zlib.crc32(repr(geo).encode()) % 1000,
                           x_dist="normal", bias=bias)
    gc.force_kernel("direct_cpasync")
    try:
        full_check(oracle_mod, d, st, pad, dil, g, "cp.async " + str(geo))
    finally:
        gc.force_kernel("auto")


# shapes the streaming kernel takes: every fast geometry, ragged tiles, several
# work items per CTA (the stage ring wraps many times), grouped and multiplied
# channels, the largest channel slices
STREAM_GEOMS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, bias
    (1, 32, 28, 28, 32, 3, 3, 1, 1, 1, 8, True),
    (3, 12, 17, 24, 12, 3, 3, 1, 1, 1, 12, True),     # ragged rows
    (2, 8, 33, 132, 8, 3, 3, 1, 1, 1, 8, False),     # two column tiles
    (1, 16, 56, 56, 32, 3, 3, 1, 1, 1, 16, False),   # channel multiplier 2
    (2, 24, 20, 20, 48, 3, 3, 1, 1, 1, 3, True),     # cpg 8, kpg 16
    (2, 16, 56, 56, 16, 3, 3, 2, 1, 1, 16, True),    # stride 2
    (1, 8, 32, 36, 8, 3, 3, 2, 1, 1, 8, False),
    (1, 8, 20, 24, 16, 3, 3, 1, 0, 1, 1, True),      # pad 0 dense
    (1, 16, 12, 40, 16, 1, 1, 1, 0, 1, 4, True),     # pointwise grouped
    (1, 64, 12, 12, 64, 3, 3, 1, 1, 1, 1, False),    # dense 3x3, 64 channels per group
    (32, 64, 56, 56, 64, 3, 3, 1, 1, 1, 64, True),   # 1024 work items: many per CTA
    (8, 256, 28, 28, 256, 3, 3, 1, 1, 1, 128, False),
    (2, 32, 112, 112, 32, 3, 3, 1, 1, 1, 8, True),   # 112-wide rows, cpg 4
    (1, 8, 64, 1028, 8, 3, 3, 2, 1, 1, 8, False),    # wide rows: column tiles, stride 2
]


@pytest.mark.parametrize("geo", STREAM_GEOMS, ids=lambda g: "x".join(map(str, g[:11])))
def test_forced_stream_matches_oracle(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=13 + zlib.crc32(repr(geo).encode()) % 1000,
                           x_dist="normal", bias=bias)
    gc.force_kernel("direct_stream")
    try:
        assert gc.plan_name(N, C, H, W, K, R, S, st, pad, dil, g).startswith("direct_stream")
        full_check(oracle_mod, d, st, pad, dil, g, "stream " + str(geo))
    finally:
        gc.force_kernel("auto")
    assert gc.library().gconv_device_error_status() == gc.OK


@pytest.mark.parametrize("geo", GEOMS[:10] + STREAM_GEOMS[10:], ids=lambda g: "x".join(map(str, g[:11])))
def test_forced_blocked_matches_oracle(oracle_mod, geo):
    """The blocked (one tile per CTA) direct kernel on shapes the dispatcher streams."""
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=17 + zlib.crc32(repr(geo).encode()) % 1000,
                           x_dist="normal", bias=bias)
    gc.force_kernel("direct_blocked")
    try:
        assert not gc.plan_name(N, C, H, W, K, R, S, st, pad, dil, g).startswith("direct_stream")
        full_check(oracle_mod, d, st, pad, dil, g, "blocked " + str(geo))
    finally:
        gc.force_kernel("auto")


def test_stream_affine_clamp_and_misaligned_output(oracle_mod):
    """Streaming kernel with the affine + clamp epilogue, y not 16-byte aligned (scalar stores)."""
    d = inputs.conv_inputs(4, 64, 56, 56, 64, 3, 3, 64, seed=4500)
    rng = torch.Generator().manual_seed(4501)
    sc = torch.rand(64, generator=rng) + 0.5
    sh = torch.randn(64, generator=rng) * 0.5
    out = Guarded((4, 64, 56, 56), misalign=1)
    gc.force_kernel("direct_stream")
    try:
        gc.conv2d_affine_clamp(d["x"].cuda(), d["w"].cuda(), sc.cuda(), sh.cuda(), 0.0, 6.0, 1, 1, 1, 64,
                               out=out.y)
        torch.cuda.synchronize()
    finally:
        gc.force_kernel("auto")
    out.check()
    ref, absacc = oracle_mod.conv2d_affine_clamp(d["x"].numpy(), d["w"].numpy(), sc.numpy(), sh.numpy(), 0.0,
                                                 6.0, 1, 1, 1, 64, return_absacc=True)
    s64 = sc.double().numpy()[None, :, None, None]
    t64 = sh.double().numpy()[None, :, None, None]
    tol = np.abs(s64) * (1e-5 * absacc + 1e-6) + 2.0 ** -23 * (np.abs(ref) + np.abs(t64)) + 1e-30
    err = np.abs(out.y.cpu().double().numpy() - ref)
    assert np.all(err <= tol), f"max err/tol {np.max(err / tol):.3g}"


# per-axis stride / padding / dilation ("Kimi-K2.6__l1_p62", padding as an (h, w) tuple)
AXIS_GEOMS = [
    # N, C, H, W, K, R, S, (sh, sw), (ph, pw), (dh, dw), groups, bias
    (2, 16, 30, 34, 16, 3, 3, (1, 2), (1, 0), (1, 1), 16, True),      # depthwise, generic kernel
    (1, 8, 21, 40, 16, 3, 5, (2, 1), (0, 2), (1, 2), 4, False),
    (2, 32, 24, 36, 64, 5, 9, (1, 1), (2, 4), (1, 1), 1, True),       # "same" 5x9: implicit GEMM
    (1, 16, 17, 29, 32, 3, 3, (1, 1), (2, 1), (2, 1), 1, False),      # implicit GEMM, dilation (2, 1)
    (1, 8, 16, 16, 8, 3, 3, (1, 1), (1, 1), (1, 1), 8, True),         # equal axes: the plain entry point
]


@pytest.mark.parametrize("geo", AXIS_GEOMS, ids=lambda g: "x".join(map(str, g[:7])) + f"_s{g[7]}_p{g[8]}_d{g[9]}")
def test_per_axis_geometry_matches_oracle(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=19 + zlib.crc32(repr(geo).encode()) % 1000,
                           x_dist="normal", bias=bias)
    ref, acc = oracle_mod.conv2d(d["x"], d["w"], d.get("bias"), st, pad, dil, g, return_absacc=True)
    out = Guarded(ref.shape)
    gc.conv2d(d["x"].cuda(), d["w"].cuda(), d["bias"].cuda() if bias else None, st, pad, dil, g, out=out.y)
    torch.cuda.synchronize()
    out.check()
    assert_conv_close(out.y.cpu().numpy(), ref, acc, "per-axis " + str(geo))


def test_per_axis_equal_values_are_bitwise_the_plain_entry_point():
    d = inputs.conv_inputs(2, 32, 28, 28, 32, 3, 3, 32, seed=4700, x_dist="normal")
    x, w = d["x"].cuda(), d["w"].cuda()
    lib = gc.library()
    a = torch.empty(2, 32, 28, 28, device="cuda")
    b = torch.empty(2, 32, 28, 28, device="cuda")
    h = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.gconv2d_fwd(x.data_ptr(), w.data_ptr(), None, 2, 32, 28, 28, 32, 3, 3, 1, 1, 1, 32,
                           a.data_ptr(), h) == gc.OK
    assert lib.gconv2d_fwd_ex(x.data_ptr(), w.data_ptr(), None, 2, 32, 28, 28, 32, 3, 3, 1, 1, 1, 1, 1, 1, 32,
                              b.data_ptr(), h) == gc.OK
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_forced_cpasync_chain(oracle_mod):
    d = inputs.chain_inputs(2, 8, 40, 40, 32, 3, 3, 1, 8, seed=64, bias_scale_std=1.0, affine="random")
    gc.force_kernel("direct_cpasync")
    try:
        y = _chain_dev(d, 1, 0, 1, 1, 1e-5).cpu().numpy()
    finally:
        gc.force_kernel("auto")
    ref = _chain_ref(oracle_mod, d, 1, 0, 1, 1, 1e-5)
    assert_chain_close(y, ref, d["scale"].numpy(), d["gamma"].numpy(), 1e-5, 4, "cp.async chain")


def test_no_device_error_flag():
    assert gc.library().gconv_device_error_status() == gc.OK


@pytest.mark.parametrize("mis", [1, 2, 3])
def test_misaligned_pointers(oracle_mod, mis):
    d = inputs.conv_inputs(2, 16, 28, 28, 16, 3, 3, 16, seed=40 + mis, x_dist="normal", bias=True)
    full_check(oracle_mod, d, 1, 1, 1, 16, f"misaligned by {mis}", misalign=mis)


def test_bias_null_equals_zero_bias():
    d = inputs.conv_inputs(2, 8, 20, 20, 8, 3, 3, 8, seed=50)
    x, w = d["x"].cuda(), d["w"].cuda()
    y0 = gc.conv2d(x, w, None, 1, 1, 1, 8)
    yz = gc.conv2d(x, w, torch.zeros(8, device="cuda"), 1, 1, 1, 8)
    torch.cuda.synchronize()
    assert torch.equal(y0, yz)


def test_delta_kernel_is_exact_identity():
    d = inputs.conv_inputs(2, 32, 56, 56, 32, 3, 3, 32, seed=51)
    w = torch.zeros(32, 1, 3, 3)
    w[:, 0, 1, 1] = 1.0
    y = gc.conv2d(d["x"].cuda(), w.cuda(), None, 1, 1, 1, 32)
    torch.cuda.synchronize()
    assert torch.equal(y.cpu(), d["x"])


def test_stream_ordering():
    """The call runs on torch's current stream (a side stream here)."""
    d = inputs.conv_inputs(4, 64, 56, 56, 64, 3, 3, 64, seed=52)
    s = torch.cuda.Stream()
    x = d["x"].cuda()
    w = d["w"].cuda()
    ref = gc.conv2d(x, w, None, 1, 1, 1, 64)
    with torch.cuda.stream(s):
        x2 = x * 1.0
        y = gc.conv2d(x2, w, None, 1, 1, 1, 64)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)


# ------------------------------------------------------------------ fused chain

def _chain_dev(d, stride, pad, dil, groups, eps):
    x = d["x"].cuda()
    w = d["w"].cuda()
    bias = (d["b_conv"] + d["b_extra"]).cuda()
    N, C, H, W = d["x"].shape
    K, _, R, S = d["w"].shape
    P, Q = gc.output_size(H, W, R, S, stride, pad, dil)
    out = Guarded((N, K, P, Q))
    gc.conv2d_bias_scale_sigmoid_groupnorm(x, w, bias, d["scale"].cuda(), d["gn_groups"],
                                           d["gamma"].cuda(), d["beta"].cuda(), eps, stride, pad,
                                           dil, groups, out=out.y)
    torch.cuda.synchronize()
    out.check()
    return out.y


def _chain_ref(oracle_mod, d, stride, pad, dil, groups, eps, pairs=None):
    return oracle_mod.chain(d["x"], d["w"], d["b_conv"], d["b_extra"], d["scale"], d["gn_groups"],
                            d["gamma"], d["beta"], eps, stride, pad, dil, groups, pairs)


CHAINS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, gn_groups, bias/scale std, affine
    (2, 8, 40, 40, 32, 3, 3, 1, 0, 1, 1, 8, 0.02, "identity"),   # the workload's geometry, small
    (2, 8, 40, 40, 32, 3, 3, 1, 0, 1, 1, 8, 1.0, "random"),      # stressed statistics
    (3, 8, 37, 45, 32, 3, 3, 1, 0, 1, 1, 8, 1.0, "random"),      # ragged tiles
    (2, 8, 24, 24, 32, 3, 3, 1, 0, 1, 1, 2, 1.0, "random"),      # 16 channels per GN group
    (2, 8, 24, 24, 32, 3, 3, 1, 0, 1, 1, 32, 1.0, "random"),     # 1 channel per GN group
    (2, 16, 30, 30, 16, 3, 3, 1, 1, 1, 16, 4, 1.0, "random"),    # depthwise conv in the chain
    (2, 12, 21, 19, 24, 3, 3, 1, 1, 1, 3, 6, 1.0, "random"),     # grouped conv, GN crosses groups
    (1, 8, 17, 17, 24, 3, 3, 2, 1, 1, 1, 3, 1.0, "random"),      # stride 2
    (1, 6, 15, 16, 12, 5, 3, 1, 1, 1, 2, 4, 1.0, "random"),      # generic geometry
    (2, 8, 40, 40, 32, 3, 3, 1, 0, 1, 1, 8, 3.0, "random"),      # saturating logistic
    (2, 8, 30, 33, 32, 3, 3, 1, 0, 1, 1, 1, 1.0, "random"),      # one group of all 32 channels
    (1, 16, 21, 22, 64, 3, 3, 1, 1, 1, 1, 4, 1.0, "random"),     # 64 channels, 16 per group
    (1, 16, 21, 22, 64, 3, 3, 1, 1, 1, 1, 1, 1.0, "random"),     # 64 channels in one group
    (1, 16, 19, 140, 64, 3, 3, 1, 1, 1, 1, 32, 1.0, "random"),   # 64 channels, 2 per group
]


@pytest.mark.parametrize("cfg", CHAINS, ids=lambda c: "x".join(map(str, c[:12])) + f"_{c[12]}")
def test_chain_full(oracle_mod, cfg):
    N, C, H, W, K, R, S, st, pad, dil, g, gn, std, affine = cfg
    d = inputs.chain_inputs(N, C, H, W, K, R, S, g, gn, seed=60 + zlib.crc32(repr(cfg).encode()) % 1000,
                            bias_scale_std=std, affine=affine)
    eps = 1e-5
    y = _chain_dev(d, st, pad, dil, g, eps).cpu().numpy()
    ref = _chain_ref(oracle_mod, d, st, pad, dil, g, eps)
    assert_chain_close(y, ref, d["scale"].numpy(), d["gamma"].numpy(), eps, K // gn, str(cfg))


def test_chain_workload_full_size_sampled_groups(oracle_mod):
    ch = wl.FUSED_CHAIN
    s = ch.conv
    d = inputs.chain_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, 1, ch.gn_groups,
                            seed=wl.SEEDS["fused_chain"])
    eps = 1e-5
    y = _chain_dev(d, 1, 0, 1, 1, eps)
    assert tuple(y.shape) == (128, 32, 254, 254)
    kgn = s.K // ch.gn_groups
    pairs = [(0, 0), (127, 7), (64, 3), (5, 6)]
    ref = _chain_ref(oracle_mod, d, 1, 0, 1, 1, eps, pairs=pairs)
    got = np.stack([y[n, G * kgn:(G + 1) * kgn].cpu().numpy() for n, G in pairs])
    sc = np.stack([d["scale"].numpy()[G * kgn:(G + 1) * kgn] for _, G in pairs])
    ga = np.stack([d["gamma"].numpy()[G * kgn:(G + 1) * kgn] for _, G in pairs])
    assert_chain_close(got, ref, sc, ga, eps, kgn, "fused chain full size")
    # every group is normalised: per (n, G) mean ~ 0 and mean square ~ var/(var+eps)
    yy = y.view(128, 8, -1).double()
    m = yy.mean(dim=2)
    assert float(m.abs().max()) < 1e-3


def test_chain_deterministic():
    d = inputs.chain_inputs(4, 8, 64, 64, 32, 3, 3, 1, 8, seed=70, bias_scale_std=1.0)
    y1 = _chain_dev(d, 1, 0, 1, 1, 1e-5).clone()
    y2 = _chain_dev(d, 1, 0, 1, 1, 1e-5)
    assert torch.equal(y1, y2)


def test_chain_scale_zero_gives_beta():
    d = inputs.chain_inputs(2, 8, 20, 20, 32, 3, 3, 1, 8, seed=71, affine="random")
    d["scale"] = torch.zeros(32)
    y = _chain_dev(d, 1, 0, 1, 1, 1e-5)
    want = d["beta"].view(1, 32, 1, 1).expand_as(y.cpu())
    assert torch.equal(y.cpu(), want.contiguous())


# ------------------------------------------------------------------ implicit GEMM (tcgen05)

IGEMM_GEOMS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, bias
    (1, 8, 20, 150, 32, 3, 3, 1, 0, 1, 1, True),      # Q > 128: two M tiles along q, ragged
    (2, 8, 19, 33, 32, 3, 3, 1, 1, 1, 1, False),      # padding, ragged rows
    (1, 16, 12, 40, 64, 5, 9, 1, 0, 1, 1, True),      # the dense asymmetric kernel
    (1, 32, 9, 137, 64, 5, 9, 1, 2, 1, 1, False),     # 5x9 with padding, Q = 133
    (1, 16, 17, 29, 32, 3, 3, 1, 2, 2, 1, True),      # dilation 2
    (2, 16, 10, 20, 64, 3, 3, 1, 1, 1, 2, True),      # two groups of 8 -> 32
    (1, 8, 9, 18, 128, 3, 3, 1, 1, 1, 1, False),      # N = 128
    (1, 8, 6, 10, 256, 3, 3, 1, 1, 1, 1, True),       # N = 256
    (1, 24, 11, 21, 32, 3, 5, 1, 1, 1, 1, False),     # R != S, three channel steps
    (1, 8, 1, 140, 32, 1, 3, 1, 0, 1, 1, True),       # single output row
    (1, 8, 13, 40, 32, 2, 3, 1, 0, 1, 1, True),       # two tap rows folded into one MMA
    (1, 16, 15, 50, 32, 5, 3, 1, 2, 1, 1, False),     # 5 tap rows: too large to fold, one per MMA
    (1, 16, 12, 30, 64, 4, 1, 1, 0, 1, 1, True),      # 4 tap rows x 64 channels: N = 256 MMAs
]


@pytest.mark.parametrize("geo", IGEMM_GEOMS, ids=lambda g: "x".join(map(str, g[:11])))
def test_igemm_matches_oracle(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=zlib.crc32(repr(geo).encode()) % 10000,
                           x_dist="normal", bias=bias)
    gc.force_kernel("igemm")
    try:
        assert gc.plan_name(N, C, H, W, K, R, S, st, pad, dil, g).startswith("igemm_tf32_bf16x")
        full_check(oracle_mod, d, st, pad, dil, g, "igemm " + str(geo))
    finally:
        gc.force_kernel("auto")
    assert gc.library().gconv_device_error_status() == gc.OK


def test_igemm_calls_back_to_back_on_one_stream(oracle_mod):
    """Two implicit-GEMM convolutions queued on one stream with different inputs
    share the workspace; stream order keeps them apart (both exact to the oracle)."""
    geo = (2, 32, 24, 36, 64, 5, 9, 1, 2, 1, 1)   # 64 output channels: the split variant (x copies in the workspace)
    N, C, H, W, K, R, S, st, pad, dil, g = geo
    d1 = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=4800, x_dist="normal", w_bound=0.05)
    d2 = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=4801, x_dist="uniform01", w_bound=0.05)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y1 = gc.conv2d(d1["x"].cuda(), d1["w"].cuda(), None, st, pad, dil, g)
        y2 = gc.conv2d(d2["x"].cuda(), d2["w"].cuda(), None, st, pad, dil, g)
    torch.cuda.synchronize()
    assert gc.plan_name(N, C, H, W, K, R, S, st, pad, dil, g).startswith("igemm")
    for d, y in ((d1, y1), (d2, y2)):
        ref, acc = oracle_mod.conv2d(d["x"], d["w"], None, st, pad, dil, g, return_absacc=True)
        assert_conv_close(y.cpu().numpy(), ref, acc, "back-to-back igemm")


def test_dense_5x9_direct_path_small(oracle_mod):
    """The CUDA-core direct path on the dense asymmetric shape (the dispatcher's alternative)."""
    d = inputs.conv_inputs(1, 32, 37, 70, 64, 5, 9, 1, 78, x_dist="uniform01",
                           w_bound=1 / math.sqrt(1440))
    gc.force_kernel("direct")
    try:
        full_check(oracle_mod, d, 1, 0, 1, 1, "direct dense 5x9 ragged")
    finally:
        gc.force_kernel("auto")


@pytest.mark.parametrize("mode", ["igemm", "direct"])
def test_chain_paths_agree_with_oracle(oracle_mod, mode):
    d = inputs.chain_inputs(2, 8, 45, 140, 32, 3, 3, 1, 8, seed=81, bias_scale_std=1.0, affine="random")
    gc.force_kernel(mode)
    try:
        y = _chain_dev(d, 1, 0, 1, 1, 1e-5).cpu().numpy()
    finally:
        gc.force_kernel("auto")
    ref = _chain_ref(oracle_mod, d, 1, 0, 1, 1, 1e-5)
    assert_chain_close(y, ref, d["scale"].numpy(), d["gamma"].numpy(), 1e-5, 4, f"{mode} chain")


_FOLD_SCRIPT = r"""
import sys, json
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import inputs
outs = {}
gc.force_kernel("igemm")
for i, geo in enumerate(json.loads(sys.argv[3])):
    N, C, H, W, K, R, S, st, pad, dil, g, seed = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=seed, x_dist="normal", bias=True)
    y = gc.conv2d(d["x"].cuda(), d["w"].cuda(), d["bias"].cuda(), st, pad, dil, g)
    outs[str(i)] = y.cpu().numpy()
d = inputs.chain_inputs(2, 8, 40, 44, 32, 3, 3, 1, 8, seed=96, bias_scale_std=1.0, affine="random")
y = gc.conv2d_bias_scale_sigmoid_groupnorm(d["x"].cuda(), d["w"].cuda(), (d["b_conv"] + d["b_extra"]).cuda(),
                                           d["scale"].cuda(), 8, d["gamma"].cuda(), d["beta"].cuda(), 1e-5,
                                           1, 0, 1, 1)
outs["chain"] = y.cpu().numpy()
np.savez(sys.argv[2], **outs)
print("ok")
"""

FOLD_GEOMS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, seed
    (2, 8, 21, 140, 32, 3, 3, 1, 1, 1, 1, 1),     # 3 tap rows x 32 channels per MMA, two column tiles
    (1, 16, 14, 40, 64, 3, 3, 1, 0, 1, 1, 2),     # 3 x 64
    (1, 8, 9, 18, 128, 3, 3, 1, 1, 1, 1, 3),      # 2 x 128 plus a one-row chunk
    (1, 32, 20, 24, 32, 3, 3, 1, 1, 1, 4, 4),     # packed groups
    (1, 8, 13, 40, 32, 2, 3, 1, 0, 1, 1, 5),      # 2 x 32
]


def test_igemm_folded_tap_rows_match_unfolded_bitwise(tmp_path):
    """One MMA per (staged row, tap column) over several tap rows' weights
    (GCONV_IGEMM_FOLD=2: plain convolutions and the chain) against one MMA per
    tap (GCONV_IGEMM_FOLD=0).  The setting is read once per process, so each
    runs in a child process.  Every output row receives the same products in
    the same order, so the bits agree."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = {}
    for fold in ("0", "2"):
        out = tmp_path / f"fold{fold}.npz"
        env = dict(os.environ, GCONV_IGEMM_FOLD=fold)
        r = subprocess.run([sys.executable, "-c", _FOLD_SCRIPT, root, str(out), json.dumps(FOLD_GEOMS)], env=env,
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
        outs[fold] = np.load(out)
    for key in outs["0"].files:
        assert np.array_equal(outs["0"][key], outs["2"][key]), key
    # the default (folded plain convolutions) in this process gives the same bits too
    gc.force_kernel("igemm")
    try:
        for i, geo in enumerate(FOLD_GEOMS):
            N, C, H, W, K, R, S, st, pad, dil, g, seed = geo
            d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=seed, x_dist="normal", bias=True)
            y = gc.conv2d(d["x"].cuda(), d["w"].cuda(), d["bias"].cuda(), st, pad, dil, g).cpu().numpy()
            assert np.array_equal(y, outs["0"][str(i)]), geo
    finally:
        gc.force_kernel("auto")


_SLICES_SCRIPT = r"""
import sys, json
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np, torch
import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import inputs
import oracle
from tolerance import assert_conv_close
gc.force_kernel("igemm")
for geo in json.loads(sys.argv[2]):
    N, C, H, W, K, R, S, st, pad, dil, g, seed = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=seed, x_dist="normal", bias=True)
    y = gc.conv2d(d["x"].cuda(), d["w"].cuda(), d["bias"].cuda(), st, pad, dil, g).cpu().numpy()
    ref, acc = oracle.conv2d(d["x"], d["w"], d["bias"], st, pad, dil, g, return_absacc=True)
    assert_conv_close(y, ref, acc, "slices " + str(geo))
print("ok")
"""


def test_igemm_folded_per_tap_column_slices_match_oracle():
    """The folded GEMM with one weight slice per tap column (off by default,
    GCONV_IGEMM_FOLD_SLICES=1, read once per process: a child process) on
    shapes whose whole-chunk slices do not fit shared memory: 5x9 at 64
    output channels (two chunks of 3 tap rows, one zero row) and 3x5 at 32."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    geos = [(1, 16, 12, 40, 64, 5, 9, 1, 0, 1, 1, 11), (1, 32, 9, 137, 64, 5, 9, 1, 2, 1, 1, 12),
            (1, 24, 11, 21, 32, 3, 5, 1, 1, 1, 1, 13), (2, 32, 20, 24, 64, 7, 7, 1, 3, 1, 1, 14)]
    env = dict(os.environ, GCONV_IGEMM_FOLD_SLICES="1")
    r = subprocess.run([sys.executable, "-c", _SLICES_SCRIPT, root, json.dumps(geos)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


# ---------------------------------------------------- fused operand staging (igemm)
# The fused implicit GEMM stages x raw by TMA and converts it in shared memory;
# the conversion is the split pass's arithmetic, so both give the same bits.
FUSED_GEOMS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, bias
    (2, 8, 19, 36, 32, 3, 3, 1, 1, 1, 1, True),       # padding 1: raw box starts left of the image
    (1, 8, 20, 152, 32, 3, 3, 1, 0, 1, 1, False),     # two column tiles, ragged
    (2, 16, 10, 20, 64, 3, 3, 1, 1, 1, 2, True),      # two groups, two channel steps
    (1, 24, 11, 24, 32, 3, 5, 1, 1, 1, 1, False),     # R != S, three channel steps
    (1, 16, 17, 32, 32, 3, 3, 1, 2, 2, 1, True),      # dilation 2, pad 2 (start not a multiple of 4)
    (2, 8, 64, 68, 32, 3, 3, 1, 3, 1, 1, True),       # pad 3
]


@pytest.mark.parametrize("geo", FUSED_GEOMS, ids=lambda g: "x".join(map(str, g[:11])))
def test_fused_igemm_matches_split_bitwise_and_oracle(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=23 + zlib.crc32(repr(geo).encode()) % 1000,
                           x_dist="normal", bias=bias)
    outs = {}
    for mode in ("igemm_fused", "igemm_split"):
        gc.force_kernel(mode)
        try:
            plan = gc.plan_name(N, C, H, W, K, R, S, st, pad, dil, g)
            assert plan == ("igemm_tf32_bf16x_fused" if mode == "igemm_fused" else "igemm_tf32_bf16x"), plan
            outs[mode] = run_conv(d, st, pad, dil, g).cpu()
        finally:
            gc.force_kernel("auto")
    assert torch.equal(outs["igemm_fused"], outs["igemm_split"])
    ref, acc = oracle_mod.conv2d(d["x"], d["w"], d.get("bias"), st, pad, dil, g, return_absacc=True)
    assert_conv_close(outs["igemm_fused"].numpy(), ref, acc, "fused " + str(geo))
    assert gc.library().gconv_device_error_status() == gc.OK


@pytest.mark.parametrize("cfg", [(2, 8, 40, 40, 32, 8, 1.0), (3, 8, 37, 44, 32, 2, 1.0), (2, 8, 24, 24, 32, 32, 3.0)])
def test_fused_chain_matches_oracle(oracle_mod, cfg):
    """Both operand stagings in the chain against the oracle.  (Their outputs
    are not compared bit for bit: the fused variant tiles 6 output rows, the
    split one 8, so the GroupNorm partial sums are rounded in other groupings.)"""
    N, C, H, W, K, gn, std = cfg
    d = inputs.chain_inputs(N, C, H, W, K, 3, 3, 1, gn, seed=90 + N * H, bias_scale_std=std, affine="random")
    ref = _chain_ref(oracle_mod, d, 1, 0, 1, 1, 1e-5)
    for mode in ("igemm_fused", "igemm_split"):
        gc.force_kernel(mode)
        try:
            assert gc.plan_name(N, C, H, W, K, 3, 3, 1, 0, 1, 1, chain=True) == (
                "igemm_tf32_bf16x_fused" if mode == "igemm_fused" else "igemm_tf32_bf16x")
            y = _chain_dev(d, 1, 0, 1, 1, 1e-5).cpu()
        finally:
            gc.force_kernel("auto")
        assert_chain_close(y.numpy(), ref, d["scale"].numpy(), d["gamma"].numpy(), 1e-5, K // gn,
                           f"{mode} chain " + str(cfg))


# groups with fewer than 32 output channels packed 32/kpg to a tensor-core tile
# (block-diagonal weights): grouped, depthwise and channel-multiplier shapes
PACKED_GEOMS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, bias
    (2, 32, 20, 24, 32, 3, 3, 1, 1, 1, 4, True),      # 8 channels per group: 4 groups per tile
    (1, 64, 16, 40, 64, 3, 3, 1, 1, 1, 8, False),     # two packed groups
    (1, 32, 14, 28, 32, 3, 3, 1, 1, 1, 8, True),      # 4 channels per group: 8 per tile
    (1, 32, 16, 32, 32, 3, 3, 1, 1, 1, 32, True),     # depthwise: 32 groups per tile
    (1, 16, 16, 24, 32, 3, 3, 1, 1, 1, 16, False),    # depthwise with channel multiplier 2
    (2, 32, 9, 140, 32, 3, 3, 1, 0, 1, 4, True),      # ragged, two column tiles
]


@pytest.mark.parametrize("geo", PACKED_GEOMS, ids=lambda g: "x".join(map(str, g[:11])))
def test_packed_groups_on_tensor_cores_match_oracle(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=29 + zlib.crc32(repr(geo).encode()) % 1000,
                           x_dist="normal", bias=bias)
    ref, acc = oracle_mod.conv2d(d["x"], d["w"], d.get("bias"), st, pad, dil, g, return_absacc=True)
    outs = {}
    for mode in ("igemm_fused", "igemm_split"):
        gc.force_kernel(mode)
        try:
            plan = gc.plan_name(N, C, H, W, K, R, S, st, pad, dil, g)
            assert plan.startswith("igemm") and plan.endswith("packed"), plan
            outs[mode] = run_conv(d, st, pad, dil, g).cpu()
        finally:
            gc.force_kernel("auto")
        assert_conv_close(outs[mode].numpy(), ref, acc, f"{mode} packed " + str(geo))
    assert torch.equal(outs["igemm_fused"], outs["igemm_split"])
    assert gc.library().gconv_device_error_status() == gc.OK


def test_packed_groups_in_the_chain(oracle_mod):
    d = inputs.chain_inputs(2, 32, 20, 24, 32, 3, 3, 4, 8, seed=97, bias_scale_std=1.0, affine="random")
    gc.force_kernel("igemm")
    try:
        assert gc.plan_name(2, 32, 20, 24, 32, 3, 3, 1, 0, 1, 4, chain=True).endswith("packed")
        y = _chain_dev(d, 1, 0, 1, 4, 1e-5).cpu().numpy()
    finally:
        gc.force_kernel("auto")
    ref = _chain_ref(oracle_mod, d, 1, 0, 1, 4, 1e-5)
    assert_chain_close(y, ref, d["scale"].numpy(), d["gamma"].numpy(), 1e-5, 4, "packed chain")


# Winograd F(2x2, 3x3) on the CUDA cores: same convolution, 16 multiplies per
# 2x2 tile and input channel; its FP32 error stays inside the conv bound
WINO_GEOMS = [
    # N, C, H, W, K, R, S, stride, pad, dil, groups, bias
    (2, 32, 20, 24, 32, 3, 3, 1, 1, 1, 4, True),      # 8 channels per group (the FP32-bound sweep case)
    (1, 64, 17, 23, 64, 3, 3, 1, 1, 1, 8, False),     # odd sizes: ragged 2x2 tiles
    (1, 16, 9, 13, 32, 3, 3, 1, 0, 1, 2, True),       # pad 0, channel multiplier 2
    (2, 8, 33, 40, 8, 3, 3, 1, 1, 1, 1, False),       # dense
    (1, 24, 15, 14, 48, 3, 3, 1, 2, 1, 3, True),      # pad 2
    (1, 8, 1, 9, 4, 3, 3, 1, 1, 1, 2, False),         # one output row, 2 channels per thread
    (4, 512, 28, 28, 512, 3, 3, 1, 1, 1, 64, False),  # a sweep shape (cpg 8)
]


@pytest.mark.parametrize("geo", WINO_GEOMS, ids=lambda g: "x".join(map(str, g[:11])))
def test_winograd_matches_oracle(oracle_mod, geo):
    N, C, H, W, K, R, S, st, pad, dil, g, bias = geo
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=31 + zlib.crc32(repr(geo).encode()) % 1000,
                           x_dist="normal", bias=bias)
    gc.force_kernel("winograd")
    try:
        assert gc.plan_name(N, C, H, W, K, R, S, st, pad, dil, g) == "winograd_f2x2_3x3"
        full_check(oracle_mod, d, st, pad, dil, g, "winograd " + str(geo))
    finally:
        gc.force_kernel("auto")


def test_winograd_affine_clamp_and_unsupported():
    d = inputs.conv_inputs(2, 32, 16, 20, 32, 3, 3, 4, seed=4900, x_dist="normal")
    x, w = d["x"].cuda(), d["w"].cuda()
    sc = torch.rand(32, device="cuda") + 0.5
    sh = torch.randn(32, device="cuda")
    ref = gc.conv2d_affine_clamp(x, w, sc, sh, 0.0, 6.0, 1, 1, 1, 4)
    gc.force_kernel("winograd")
    try:
        y = gc.conv2d_affine_clamp(x, w, sc, sh, 0.0, 6.0, 1, 1, 1, 4)
        torch.cuda.synchronize()
        # depthwise (one channel per group) and stride 2 are not Winograd shapes: refused, not rerouted
        assert gc.plan_name(1, 8, 16, 16, 8, 3, 3, 1, 1, 1, 8) == "unsupported"
        with pytest.raises(gc.GconvError) as e:
            gc.conv2d(x, w, None, 2, 1, 1, 4)
        assert e.value.status == gc.ERR_UNSUPPORTED
    finally:
        gc.force_kernel("auto")
    assert float((y - ref).abs().max()) < 1e-3 and float(y.min()) >= 0 and float(y.max()) <= 6


_STORE_DESIGN_SCRIPT = r"""
import sys, json
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np, torch
import depthwise_convolution_fp32_b200 as gc
from depthwise_convolution_fp32_b200 import inputs
import oracle
from tolerance import assert_chain_close
d = inputs.chain_inputs(2, 8, 40, 44, 32, 3, 3, 1, 8, seed=95, bias_scale_std=1.0, affine="random")
y = gc.conv2d_bias_scale_sigmoid_groupnorm(d["x"].cuda(), d["w"].cuda(), (d["b_conv"] + d["b_extra"]).cuda(),
                                           d["scale"].cuda(), 8, d["gamma"].cuda(), d["beta"].cuda(), 1e-5,
                                           1, 0, 1, 1)
torch.cuda.synchronize()
y = y.cpu()
ref = oracle.chain(d["x"], d["w"], d["b_conv"], d["b_extra"], d["scale"], 8, d["gamma"], d["beta"], 1e-5, 1, 0, 1, 1)
assert_chain_close(y.numpy(), ref, d["scale"].numpy(), d["gamma"].numpy(), 1e-5, 4, "store design")
np.save(sys.argv[2], y.numpy())
print("ok")
"""


def test_chain_store_design_matches_recompute_bitwise(tmp_path):
    """The chain's other design (GEMM stores the logistic output, a streaming
    pass normalizes it) gives the same bits as the default (GEMM twice:
    statistics, then the normalized output); the design is chosen once per
    process, so the other one runs in a child process."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = tmp_path / "store.npy"
    env = dict(os.environ, GCONV_CHAIN_DESIGN="store")
    r = subprocess.run([sys.executable, "-c", _STORE_DESIGN_SCRIPT, root, str(out)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
    d = inputs.chain_inputs(2, 8, 40, 44, 32, 3, 3, 1, 8, seed=95, bias_scale_std=1.0, affine="random")
    y = _chain_dev(d, 1, 0, 1, 1, 1e-5).cpu().numpy()
    assert np.array_equal(y, np.load(out))


# ------------------------------------------------------------ affine + clamp epilogue
AFFINE_CASES = [
    # (N, C, H, W, K, R, S, stride, pad, dil, groups, lo, hi)
    (4, 144, 56, 56, 144, 3, 3, 1, 1, 1, 144, 0.0, 6.0),            # the depthwise workload + BN + ReLU6
    (2, 32, 14, 14, 32, 3, 3, 1, 1, 1, 16, -0.5, 0.5),               # W=14: 8-byte cp.async staging
    (2, 32, 36, 40, 64, 3, 3, 1, 1, 1, 1, 0.0, 6.0),                 # implicit GEMM
    (2, 32, 36, 40, 64, 3, 3, 1, 1, 1, 1, -math.inf, math.inf),      # implicit GEMM, no clamp
    (1, 24, 19, 23, 48, 3, 3, 2, 1, 1, 24, 0.0, 6.0),                # stride 2, channel multiplier 2
]


@pytest.mark.parametrize("case", AFFINE_CASES)
def test_affine_clamp_matches_oracle(oracle_mod, case):
    N, C, H, W, K, R, S, st, pad, dil, g, lo, hi = case
    d = inputs.conv_inputs(N, C, H, W, K, R, S, g, seed=4000 + N * C + K)
    rng = torch.Generator().manual_seed(4100 + K)
    sc = torch.rand(K, generator=rng) + 0.5
    sh = torch.randn(K, generator=rng) * 0.5
    y = gc.conv2d_affine_clamp(d["x"].cuda(), d["w"].cuda(), sc.cuda(), sh.cuda(), lo, hi, st, pad, dil, g)
    torch.cuda.synchronize()
    ref, absacc = oracle_mod.conv2d_affine_clamp(d["x"].numpy(), d["w"].numpy(), sc.numpy(), sh.numpy(), lo, hi,
                                                 st, pad, dil, g, return_absacc=True)
    s64 = sc.double().numpy()[None, :, None, None]
    t64 = sh.double().numpy()[None, :, None, None]
    # conv bound scaled by |scale|, plus one FP32 rounding of acc*scale + shift; the clamp is 1-Lipschitz
    tol = np.abs(s64) * (1e-5 * absacc + 1e-6) + 2.0 ** -23 * (np.abs(ref) + np.abs(t64)) + 1e-30
    err = np.abs(y.cpu().double().numpy() - ref)
    assert np.all(err <= tol), f"max err/tol {np.max(err / tol):.3g}"
    assert float(y.min()) >= lo and float(y.max()) <= hi


def test_affine_without_scale_shift_or_clamp_is_plain_conv():
    d = inputs.conv_inputs(2, 144, 28, 28, 144, 3, 3, 144, seed=4200)
    x, w = d["x"].cuda(), d["w"].cuda()
    a = gc.conv2d_affine_clamp(x, w, None, None, -math.inf, math.inf, 1, 1, 1, 144)
    b = gc.conv2d(x, w, None, 1, 1, 1, 144)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_device_error_status_after_calls_on_a_stream():
    # no bounded wait gives up on valid work: both status queries report OK
    lib = gc.library()
    d = inputs.conv_inputs(4, 144, 56, 56, 144, 3, 3, 144, seed=4300)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gc.conv2d(d["x"].cuda(), d["w"].cuda(), None, 1, 1, 1, 144)
    assert lib.gconv_get_last_device_error(ctypes.c_void_p(s.cuda_stream)) == gc.OK
    assert lib.gconv_device_error_status() == gc.OK
