"""Pins for the FP64 oracle: each check ties the oracle to something other than
itself -- sizes the pages state, closed forms, invariants of the definition,
an independent numpy restatement on tiny inputs, and float64 library routines.
A plausible slip in the oracle (a flipped kernel, a wrong group offset, a
dropped padding term, a Bessel-corrected variance, eps outside the square
root, bias after scale) fails at least one test here."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from depthwise_convolution_fp32_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tconv(x, w, b=None, stride=1, pad=0, dil=1, groups=1):
    t = lambda a: None if a is None else torch.from_numpy(np.asarray(a, dtype=np.float32)).double()
    return F.conv2d(t(x), t(w), t(b), stride, pad, dil, groups).numpy()


def _numpy_conv(x, w, stride, pad, dil, groups):
    """Independent restatement: pad, then sum strided slices tap by tap."""
    N, C, H, W = x.shape
    K, cpg, R, S = w.shape
    P = (H + 2 * pad - dil * (R - 1) - 1) // stride + 1
    Q = (W + 2 * pad - dil * (S - 1) - 1) // stride + 1
    xp = np.zeros((N, C, H + 2 * pad, W + 2 * pad))
    xp[:, :, pad:pad + H, pad:pad + W] = x
    y = np.zeros((N, K, P, Q))
    kpg = K // groups
    for k in range(K):
        gi = k // kpg
        for c in range(cpg):
            for r in range(R):
                for s in range(S):
                    sl = xp[:, gi * cpg + c,
                            r * dil: r * dil + (P - 1) * stride + 1: stride,
                            s * dil: s * dil + (Q - 1) * stride + 1: stride]
                    y[:, k] += float(w[k, c, r, s]) * sl
    return y


def test_output_sizes_from_pages(oracle_mod):
    cases = json.load(open(os.path.join(GOLDEN, "output_sizes.json")))["cases"]
    for c in cases:
        assert oracle_mod.out_extent(c["H"], c["R"], c["stride"], c["pad"], c["dil"]) == c["P"], c
        assert oracle_mod.out_extent(c["W"], c["S"], c["stride"], c["pad"], c["dil"]) == c["Q"], c


def test_output_size_closed_form(oracle_mod):
    for n in range(1, 20):
        for k in range(1, 6):
            for s in range(1, 4):
                for p in range(0, 3):
                    for d in range(1, 3):
                        span = n + 2 * p - d * (k - 1) - 1
                        want = span // s + 1 if span >= 0 else 0
                        assert oracle_mod.out_extent(n, k, s, p, d) == want
    # stride 2 halves a padded 3x3: 56 -> 28, 112 -> 56
    assert oracle_mod.out_extent(56, 3, 2, 1, 1) == 28
    assert oracle_mod.out_extent(112, 3, 2, 1, 1) == 56


def test_delta_kernel_is_identity(oracle_mod):
    g = inputs.generator(1)
    x = inputs.normal((2, 5, 9, 11), 1.0, g)
    for R, S in [(3, 3), (5, 9), (1, 1), (7, 3)]:
        w = np.zeros((5, 1, R, S), np.float32)
        w[:, 0, (R - 1) // 2, (S - 1) // 2] = 1.0
        y = oracle_mod.conv2d(x, w, None, 1, ((R - 1) // 2, (S - 1) // 2), 1, 5)
        np.testing.assert_array_equal(y, x.numpy().astype(np.float64))


def test_shifted_delta_is_shift_with_zero_fill(oracle_mod):
    g = inputs.generator(2)
    x = inputs.normal((1, 3, 8, 10), 1.0, g).numpy()
    # tap (r, s) = (0, 2) of a 3x3 with pad 1 reads x[p-1, q+1]
    w = np.zeros((3, 1, 3, 3), np.float32)
    w[:, 0, 0, 2] = 1.0
    y = oracle_mod.conv2d(x, w, None, 1, 1, 1, 3)
    want = np.zeros_like(y)
    want[:, :, 1:, :-1] = x[:, :, :-1, 1:]
    np.testing.assert_array_equal(y, want)


def test_all_ones_counts_in_bounds_taps(oracle_mod):
    for (H, W, R, S, st, pad, dil) in [(7, 9, 3, 3, 1, 1, 1), (6, 6, 5, 9, 1, 4, 1),
                                       (10, 11, 3, 3, 2, 1, 1), (9, 9, 3, 3, 1, 2, 2)]:
        x = np.ones((1, 2, H, W), np.float32)
        w = np.ones((2, 1, R, S), np.float32)
        y = oracle_mod.conv2d(x, w, None, st, pad, dil, 2)
        P, Q = y.shape[2:]
        for p in range(P):
            nr = sum(1 for r in range(R) if 0 <= p * st - pad + r * dil < H)
            for q in range(Q):
                ns = sum(1 for s in range(S) if 0 <= q * st - pad + s * dil < W)
                assert y[0, 0, p, q] == nr * ns and y[0, 1, p, q] == nr * ns


def test_numpy_restatement_tiny(oracle_mod):
    rng = np.random.default_rng(5)
    for (N, C, H, W, K, R, S, st, pad, dil, g) in [
            (1, 8, 16, 16, 8, 3, 3, 1, 1, 1, 4),     # the tiny grouped workload
            (2, 4, 7, 5, 6, 3, 2, 1, 0, 1, 2),
            (1, 6, 9, 9, 6, 3, 3, 2, 1, 1, 6),
            (2, 3, 8, 13, 4, 5, 9, 1, 4, 1, 1),
            (1, 4, 11, 10, 8, 3, 3, 1, 2, 2, 2),
            (1, 2, 5, 5, 4, 1, 1, 1, 0, 1, 2)]:
        x = rng.standard_normal((N, C, H, W)).astype(np.float32)
        w = rng.standard_normal((K, C // g, R, S)).astype(np.float32)
        y = oracle_mod.conv2d(x, w, None, st, pad, dil, g)
        want = _numpy_conv(x, w, st, pad, dil, g)
        np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_library_float64_conv(oracle_mod):
    rng = np.random.default_rng(6)
    for (N, C, H, W, K, R, S, st, pad, dil, g, bias) in [
            (2, 16, 14, 14, 16, 3, 3, 1, 1, 1, 16, False),
            (3, 16, 15, 17, 32, 3, 3, 1, 1, 1, 4, True),
            (1, 8, 20, 21, 8, 3, 3, 2, 1, 1, 8, False),
            (1, 6, 13, 19, 12, 5, 9, 1, 0, 1, 1, True),
            (2, 8, 12, 12, 16, 3, 3, 1, 2, 2, 2, False),
            (1, 4, 9, 9, 8, 7, 7, 1, 3, 1, 4, True)]:
        x = rng.standard_normal((N, C, H, W)).astype(np.float32)
        w = rng.standard_normal((K, C // g, R, S)).astype(np.float32)
        b = rng.standard_normal(K).astype(np.float32) if bias else None
        y = oracle_mod.conv2d(x, w, b, st, pad, dil, g)
        np.testing.assert_allclose(y, _tconv(x, w, b, st, pad, dil, g), rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- per-axis geometry
# ("Kimi-K2.6__l1_p62", ModelNew.forward: padding, stride and dilation as (h, w)
# tuples).  Each check takes different values on the two axes, so an axis mix-up
# (the W index reading the H padding, swapped strides) fails it.

def test_per_axis_all_ones_counts_in_bounds_taps(oracle_mod):
    for (H, W, R, S, sh, sw, ph, pw, dh, dw) in [(9, 12, 3, 5, 1, 2, 0, 2, 1, 1), (11, 8, 5, 3, 2, 1, 3, 0, 1, 2),
                                                 (7, 13, 3, 3, 1, 1, 1, 0, 2, 1), (12, 12, 1, 3, 3, 1, 0, 1, 1, 3)]:
        x = np.ones((1, 2, H, W), np.float32)
        w = np.ones((2, 1, R, S), np.float32)
        y = oracle_mod.conv2d(x, w, None, (sh, sw), (ph, pw), (dh, dw), 2)
        P, Q = y.shape[2:]
        assert P == (H + 2 * ph - dh * (R - 1) - 1) // sh + 1 and Q == (W + 2 * pw - dw * (S - 1) - 1) // sw + 1
        for p in range(P):
            nr = sum(1 for r in range(R) if 0 <= p * sh - ph + r * dh < H)
            for q in range(Q):
                ns = sum(1 for s_ in range(S) if 0 <= q * sw - pw + s_ * dw < W)
                assert y[0, 0, p, q] == nr * ns and y[0, 1, p, q] == nr * ns, (p, q)


def test_per_axis_shifted_delta_is_shift(oracle_mod):
    g = inputs.generator(3)
    x = inputs.normal((1, 2, 9, 14), 1.0, g).numpy()
    # a 3x5 kernel, padding (1, 2), tap (r, s) = (2, 0): y[p, q] = x[p + 1, q - 2] (zero outside)
    w = np.zeros((2, 1, 3, 5), np.float32)
    w[:, 0, 2, 0] = 1.0
    y = oracle_mod.conv2d(x, w, None, 1, (1, 2), 1, 2)
    want = np.zeros_like(y)
    want[:, :, :-1, 2:] = x[:, :, 1:, :-2]
    np.testing.assert_array_equal(y, want)
    # strides (2, 3) with the centre tap of a 3x3 and padding (1, 1): y[p, q] = x[2p, 3q]
    w = np.zeros((2, 1, 3, 3), np.float32)
    w[:, 0, 1, 1] = 1.0
    y = oracle_mod.conv2d(x, w, None, (2, 3), 1, 1, 2)
    np.testing.assert_array_equal(y, x[:, :, ::2, ::3][:, :, :y.shape[2], :y.shape[3]].astype(np.float64))


def test_per_axis_library_float64_conv(oracle_mod):
    rng = np.random.default_rng(8)
    for (N, C, H, W, K, R, S, st, pad, dil, g, bias) in [
            (2, 8, 15, 17, 8, 3, 3, (1, 2), (1, 0), (1, 1), 8, False),
            (1, 6, 13, 19, 12, 5, 9, (1, 1), (2, 4), (1, 1), 1, True),     # "same" padding of the 5x9 kernel
            (2, 8, 14, 12, 16, 3, 3, (2, 1), (0, 1), (2, 1), 2, True),
            (1, 4, 10, 16, 8, 3, 5, (1, 3), (2, 1), (1, 2), 4, False)]:
        x = rng.standard_normal((N, C, H, W)).astype(np.float32)
        w = rng.standard_normal((K, C // g, R, S)).astype(np.float32)
        b = rng.standard_normal(K).astype(np.float32) if bias else None
        y = oracle_mod.conv2d(x, w, b, st, pad, dil, g)
        np.testing.assert_allclose(y, _tconv(x, w, b, st, pad, dil, g), rtol=1e-11, atol=1e-11)


def test_per_axis_same_padding_of_the_5x9_kernel(oracle_mod):
    # the dense transcript's 512x512 input and (5, 9) kernel: padding (2, 4) keeps 512x512
    assert oracle_mod.out_extent(512, 5, 1, 2, 1) == 512 and oracle_mod.out_extent(512, 9, 1, 4, 1) == 512
    x = np.ones((1, 1, 6, 10), np.float32)
    w = np.ones((1, 1, 5, 9), np.float32)
    y = oracle_mod.conv2d(x, w, None, 1, (2, 4), 1, 1)
    assert y.shape == (1, 1, 6, 10)
    assert y[0, 0, 2, 4] == 5 * 9 and y[0, 0, 0, 0] == 3 * 5


def test_grouped_equals_concatenated_dense(oracle_mod):
    rng = np.random.default_rng(7)
    N, C, H, W, K, g = 2, 12, 9, 10, 18, 3
    x = rng.standard_normal((N, C, H, W)).astype(np.float32)
    w = rng.standard_normal((K, C // g, 3, 3)).astype(np.float32)
    y = oracle_mod.conv2d(x, w, None, 1, 1, 1, g)
    cpg, kpg = C // g, K // g
    for gi in range(g):
        part = oracle_mod.conv2d(x[:, gi * cpg:(gi + 1) * cpg], w[gi * kpg:(gi + 1) * kpg],
                                 None, 1, 1, 1, 1)
        np.testing.assert_array_equal(y[:, gi * kpg:(gi + 1) * kpg], part)


def test_depthwise_is_per_channel_correlation(oracle_mod):
    rng = np.random.default_rng(8)
    x = rng.standard_normal((2, 5, 8, 7)).astype(np.float32)
    w = rng.standard_normal((5, 1, 3, 3)).astype(np.float32)
    y = oracle_mod.conv2d(x, w, None, 1, 1, 1, 5)
    for c in range(5):
        single = oracle_mod.conv2d(x[:, c:c + 1], w[c:c + 1], None, 1, 1, 1, 1)
        np.testing.assert_array_equal(y[:, c:c + 1], single)
    # groups=1 with one channel reduces to the same thing
    np.testing.assert_allclose(y, _tconv(x, w, None, 1, 1, 1, 5), rtol=1e-12, atol=1e-12)


def test_bias_null_equals_zero_bias_and_bias_only(oracle_mod):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 4, 6, 6)).astype(np.float32)
    w = rng.standard_normal((4, 2, 3, 3)).astype(np.float32)
    y0 = oracle_mod.conv2d(x, w, None, 1, 1, 1, 2)
    yz = oracle_mod.conv2d(x, w, np.zeros(4, np.float32), 1, 1, 1, 2)
    np.testing.assert_array_equal(y0, yz)
    b = np.array([1.5, -2.0, 0.25, 3.0], np.float32)
    yb = oracle_mod.conv2d(x, np.zeros_like(w), b, 1, 1, 1, 2)
    np.testing.assert_array_equal(yb, np.broadcast_to(b.reshape(1, 4, 1, 1), yb.shape))


def test_linearity_and_channel_permutation(oracle_mod):
    rng = np.random.default_rng(10)
    x1 = rng.standard_normal((1, 6, 7, 8)).astype(np.float32)
    x2 = rng.standard_normal((1, 6, 7, 8)).astype(np.float32)
    w = rng.standard_normal((6, 6, 3, 3)).astype(np.float32)
    y = oracle_mod.conv2d(x1 + 2 * x2, w, None, 1, 1, 1, 1)
    y1 = oracle_mod.conv2d(x1, w, None, 1, 1, 1, 1)
    y2 = oracle_mod.conv2d(x2, w, None, 1, 1, 1, 1)
    np.testing.assert_allclose(y, y1 + 2 * y2, rtol=1e-5, atol=1e-5)
    perm = rng.permutation(6)
    yp = oracle_mod.conv2d(x1[:, perm], w[:, perm], None, 1, 1, 1, 1)
    np.testing.assert_allclose(yp, y1, rtol=1e-12, atol=1e-12)


def test_absacc_is_conv_of_magnitudes(oracle_mod):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((2, 8, 9, 9)).astype(np.float32)
    w = rng.standard_normal((8, 4, 3, 3)).astype(np.float32)
    b = rng.standard_normal(8).astype(np.float32)
    _, acc = oracle_mod.conv2d(x, w, b, 1, 1, 1, 2, return_absacc=True)
    want = _tconv(np.abs(x), np.abs(w), np.abs(b), 1, 1, 1, 2)
    np.testing.assert_allclose(acc, want, rtol=1e-12, atol=1e-12)


def test_point_evaluation_matches_full(oracle_mod):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((2, 6, 11, 13)).astype(np.float32)
    w = rng.standard_normal((9, 2, 5, 3)).astype(np.float32)
    b = rng.standard_normal(9).astype(np.float32)
    y, acc = oracle_mod.conv2d(x, w, b, 2, 2, 1, 3, return_absacc=True)
    idx = rng.choice(y.size, 50, replace=False)
    v, a = oracle_mod.conv2d_at(x, w, idx, b, 2, 2, 1, 3)
    np.testing.assert_array_equal(v, y.reshape(-1)[idx])
    np.testing.assert_array_equal(a, acc.reshape(-1)[idx])


def test_rejects_invalid_geometry(oracle_mod):
    x = np.zeros((1, 4, 4, 4), np.float32)
    with pytest.raises(ValueError):
        oracle_mod.conv2d(x, np.zeros((4, 4, 7, 7), np.float32), None, 1, 0, 1, 1)
    with pytest.raises(ValueError):
        oracle_mod.conv2d(x, np.zeros((4, 3, 3, 3), np.float32), None, 1, 1, 1, 1)


# ---------------------------------------------------------------- chain

def _torch_chain(d, stride=1, pad=0, dil=1, groups=1, eps=1e-5):
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float32)).double()
    z = F.conv2d(t(d["x"]), t(d["w"]), t(d["b_conv"]), stride, pad, dil, groups)
    z = z + t(d["b_extra"]).view(1, -1, 1, 1)
    a = torch.sigmoid(z * t(d["scale"]).view(1, -1, 1, 1))
    y = F.group_norm(a, d["gn_groups"], t(d["gamma"]), t(d["beta"]), eps)
    return a.numpy(), y.numpy()


def _chain(oracle_mod, d, stride=1, pad=0, dil=1, groups=1, eps=1e-5, pairs=None):
    return oracle_mod.chain(d["x"], d["w"], d["b_conv"], d["b_extra"], d["scale"],
                            d["gn_groups"], d["gamma"], d["beta"], eps,
                            stride, pad, dil, groups, pairs)


@pytest.mark.parametrize("std,affine", [(0.02, "identity"), (1.0, "random"), (3.0, "random")])
def test_chain_matches_float64_library(oracle_mod, std, affine):
    d = inputs.chain_inputs(2, 8, 20, 18, 32, 3, 3, 1, 8, seed=20, bias_scale_std=std,
                            affine=affine)
    out = _chain(oracle_mod, d)
    a, y = _torch_chain(d)
    np.testing.assert_allclose(out["a"], a, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(out["y"], y, rtol=1e-9, atol=1e-9)


def test_chain_grouped_conv_with_padding(oracle_mod):
    d = inputs.chain_inputs(2, 8, 9, 11, 12, 3, 3, 2, 3, seed=21, bias_scale_std=1.0,
                            affine="random")
    out = _chain(oracle_mod, d, pad=1, groups=2)
    _, y = _torch_chain(d, pad=1, groups=2)
    np.testing.assert_allclose(out["y"], y, rtol=1e-9, atol=1e-9)


def test_chain_scale_zero_gives_beta(oracle_mod):
    d = inputs.chain_inputs(1, 4, 8, 8, 8, 3, 3, 1, 2, seed=22, affine="random")
    d["scale"] = np.zeros(8, np.float32)
    out = _chain(oracle_mod, d)
    assert np.all(out["a"] == 0.5)
    assert np.all(out["var"] == 0.0) and np.all(out["mean"] == 0.5)
    np.testing.assert_array_equal(out["y"], np.broadcast_to(
        d["beta"].numpy().astype(np.float64).reshape(1, 8, 1, 1), out["y"].shape))


def test_chain_groupnorm_closed_forms(oracle_mod):
    d = inputs.chain_inputs(3, 8, 12, 12, 16, 3, 3, 1, 4, seed=23, bias_scale_std=1.0)
    eps = 1e-5
    out = _chain(oracle_mod, d, eps=eps)
    y = out["y"].reshape(3, 4, -1)
    var = out["var"]
    # with gamma=1, beta=0: each group has zero mean and mean square var/(var+eps)
    np.testing.assert_allclose(y.mean(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(axis=2), var / (var + eps), rtol=1e-10)
    # and the statistics are the population moments of a
    a = out["a"].reshape(3, 4, -1)
    np.testing.assert_allclose(out["mean"], a.mean(axis=2), rtol=1e-14)
    np.testing.assert_allclose(var, a.var(axis=2, ddof=0), rtol=1e-10)


def test_chain_sigmoid_symmetry(oracle_mod):
    d = inputs.chain_inputs(1, 4, 7, 9, 8, 3, 3, 1, 2, seed=24, bias_scale_std=1.5)
    out = _chain(oracle_mod, d)
    d2 = dict(d)
    d2["scale"] = -d["scale"]
    out2 = _chain(oracle_mod, d2)
    np.testing.assert_allclose(out["a"] + out2["a"], 1.0, atol=1e-15)
    # GroupNorm of 1-a is -GroupNorm(a) when gamma=1, beta=0
    np.testing.assert_allclose(out2["y"], -out["y"], atol=1e-9)


def test_chain_bias_before_scale(oracle_mod):
    """Model order: z + bias, then * scale.  With w = 0 and no conv bias,
    a = sigmoid(b_extra * scale) exactly."""
    d = inputs.chain_inputs(1, 2, 5, 5, 4, 3, 3, 1, 2, seed=25, bias_scale_std=1.0)
    d["w"] = np.zeros((4, 2, 3, 3), np.float32)
    d["b_conv"] = np.zeros(4, np.float32)
    out = _chain(oracle_mod, d)
    v = d["b_extra"].double().numpy() * d["scale"].double().numpy()
    want = 1.0 / (1.0 + np.exp(-v))
    np.testing.assert_allclose(out["a"][0, :, 0, 0], want, rtol=1e-15)


def test_chain_selected_pairs_match_full(oracle_mod):
    d = inputs.chain_inputs(3, 8, 10, 10, 16, 3, 3, 1, 4, seed=26, bias_scale_std=1.0,
                            affine="random")
    full = _chain(oracle_mod, d)
    pairs = [(2, 1), (0, 3), (1, 0)]
    part = _chain(oracle_mod, d, pairs=pairs)
    for i, (n, G) in enumerate(pairs):
        np.testing.assert_array_equal(part["y"][i], full["y"][n, G * 4:(G + 1) * 4])
        np.testing.assert_array_equal(part["a"][i], full["a"][n, G * 4:(G + 1) * 4])
        assert part["mean"][i] == full["mean"][n, G]
        assert part["var"][i] == full["var"][n, G]


def test_chain_extreme_values_are_finite(oracle_mod):
    d = inputs.chain_inputs(1, 4, 6, 6, 4, 3, 3, 1, 1, seed=27, bias_scale_std=1.0)
    d["scale"] = np.array([1e4, -1e4, 50.0, -800.0], np.float32)
    out = _chain(oracle_mod, d)
    assert np.all(np.isfinite(out["a"])) and np.all(np.isfinite(out["y"]))
    assert np.all((out["a"] >= 0) & (out["a"] <= 1))


# ---------------------------------------------------------------- affine + clamp epilogue

def test_affine_clamp_identity_is_conv(oracle_mod):
    rng = np.random.default_rng(71)
    x = rng.standard_normal((2, 6, 9, 11)).astype(np.float32)
    w = rng.standard_normal((6, 3, 3, 3)).astype(np.float32)
    a = oracle_mod.conv2d_affine_clamp(x, w, None, None, -np.inf, np.inf, 1, 1, 1, 2)
    np.testing.assert_array_equal(a, oracle_mod.conv2d(x, w, None, 1, 1, 1, 2))


def test_affine_clamp_relu6_closed_form(oracle_mod):
    # all-ones depthwise 3x3, pad 1: conv = in-bounds tap count (4 corner, 6 edge, 9 inside);
    # scale 1, shift -5, ReLU6 -> clip(count - 5, 0, 6) = 0, 1, 4
    x = np.ones((1, 2, 5, 7), np.float32)
    w = np.ones((2, 1, 3, 3), np.float32)
    y = oracle_mod.conv2d_affine_clamp(x, w, np.ones(2, np.float32), np.full(2, -5.0, np.float32),
                                       0.0, 6.0, 1, 1, 1, 2)
    assert np.all(y[:, :, 0, 0] == 0.0) and np.all(y[:, :, 0, 3] == 1.0) and np.all(y[:, :, 2, 3] == 4.0)
    # scale 2, shift 0: 2*count clipped at 6 -> 6 everywhere (counts >= 4)
    y2 = oracle_mod.conv2d_affine_clamp(x, w, np.full(2, 2.0, np.float32), None, 0.0, 6.0, 1, 1, 1, 2)
    assert np.all(y2 == 6.0)


def test_affine_is_folded_batchnorm(oracle_mod):
    # conv -> BatchNorm (inference) equals conv * scale + shift with the folded constants
    rng = np.random.default_rng(72)
    x = rng.standard_normal((2, 4, 8, 8)).astype(np.float32)
    w = rng.standard_normal((4, 1, 3, 3)).astype(np.float32)
    gamma, beta = rng.uniform(0.5, 1.5, 4), rng.normal(0, 0.1, 4)
    mean, var, eps = rng.normal(0, 0.1, 4), rng.uniform(0.5, 1.5, 4), 1e-5
    c = oracle_mod.conv2d(x, w, None, 1, 1, 1, 4)
    bn = (c - mean[None, :, None, None]) / np.sqrt(var[None, :, None, None] + eps) * gamma[None, :, None, None] \
        + beta[None, :, None, None]
    sc = (gamma / np.sqrt(var + eps)).astype(np.float32)
    sh = (beta - mean * (gamma / np.sqrt(var + eps))).astype(np.float32)
    y = oracle_mod.conv2d_affine_clamp(x, w, sc, sh, -np.inf, np.inf, 1, 1, 1, 4)
    # the folded constants are rounded to FP32 once (|rel| <= 2^-24)
    assert np.max(np.abs(y - bn)) <= 1e-6 * (1 + np.max(np.abs(bn)))


def test_affine_clamp_bounds_and_passthrough(oracle_mod):
    rng = np.random.default_rng(73)
    x = rng.standard_normal((1, 8, 10, 10)).astype(np.float32)
    w = rng.standard_normal((8, 2, 3, 3)).astype(np.float32)
    sc, sh = rng.standard_normal(8).astype(np.float32), rng.standard_normal(8).astype(np.float32)
    free = oracle_mod.conv2d_affine_clamp(x, w, sc, sh, -np.inf, np.inf, 1, 1, 1, 4)
    y = oracle_mod.conv2d_affine_clamp(x, w, sc, sh, -0.5, 0.75, 1, 1, 1, 4)
    assert y.min() >= -0.5 and y.max() <= 0.75
    inside = (free >= -0.5) & (free <= 0.75)
    assert inside.any() and (~inside).any()
    np.testing.assert_array_equal(y[inside], free[inside])
    np.testing.assert_array_equal(y[free < -0.5], -0.5)
    np.testing.assert_array_equal(y[free > 0.75], 0.75)
