"""Per-element error bounds used by the parity tests.

Convolution (stated bound): |y_gpu - y_oracle| <= 1e-5 * sum|w*x| + 1e-6, where
sum|w*x| (the oracle's ``absacc``) also counts |bias|.

Fused chain (derived here, step by step, from the convolution bound; the
oracle supplies every exact value):
  z      : tau_z = 1e-5 * absacc + 1e-6                      (conv + folded bias)
  a      : tau_a = |scale_k| / 4 * tau_z + 3e-7              (the logistic function
           is 1/4-Lipschitz; 3e-7 ~ 5 ulp at 0.5 covers expf, the division and
           the FP32 rounding of a)
  mu     : tau_mu = max tau_a over the group + 1e-7          (a mean of values
           each within tau_a; 1e-7 for the FP32 rounding of mu)
  var    : tau_v = 2 * max|a - mu| * max tau_a + (max tau_a)^2 + 1e-6 * var + 1e-12
  y      : with rstd = 1/sqrt(var + eps),
           tau_y = |gamma| * rstd * (tau_a + tau_mu)
                 + |gamma| * |a - mu| * rstd * tau_v / (2 * (var + eps))
                 + 2e-6 * (1 + |y|)
The last term covers the FP32 rounding of rstd*gamma, of the product and of
the affine add.
"""
from __future__ import annotations

import numpy as np


def conv_tol(absacc):
    return 1e-5 * np.asarray(absacc) + 1e-6


def assert_conv_close(y_gpu, y_ref, absacc, what=""):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - y_ref)
    tol = conv_tol(absacc)
    bad = ~(err <= tol)          # NaN counts as bad
    if bad.any():
        i = np.flatnonzero(bad.reshape(-1))[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside 1e-5*sum|wx|+1e-6; "
            f"max err/tol = {np.nanmax(err / tol):.3g}; first flat indices {i.tolist()} "
            f"gpu={y_gpu.reshape(-1)[i].tolist()} ref={np.asarray(y_ref).reshape(-1)[i].tolist()}")
    return float(np.max(err / tol)) if err.size else 0.0


def chain_tols(ref, scale, gamma, eps, kgn):
    """Return (tau_a, tau_y) arrays shaped like ref['y'] ([groups, kgn, P, Q]
    or [N, K, P, Q]); scale/gamma are per output channel of that layout."""
    a = ref["a"]
    shp = a.shape
    if a.ndim == 4 and ref["mean"].ndim == 2:                    # full [N,K,P,Q]
        N, K = shp[0], shp[1]
        G = K // kgn
        a_g = a.reshape(N, G, kgn, -1)
        acc = ref["absacc"].reshape(N, G, kgn, -1)
        sc = np.abs(np.asarray(scale, np.float64)).reshape(1, G, kgn, 1)
        ga = np.abs(np.asarray(gamma, np.float64)).reshape(1, G, kgn, 1)
        mu = ref["mean"].reshape(N, G, 1, 1)
        var = ref["var"].reshape(N, G, 1, 1)
    else:                                                        # selected groups
        npairs = shp[0]
        a_g = a.reshape(npairs, 1, kgn, -1)
        acc = ref["absacc"].reshape(npairs, 1, kgn, -1)
        sc = np.abs(np.asarray(scale, np.float64)).reshape(npairs, 1, kgn, 1)
        ga = np.abs(np.asarray(gamma, np.float64)).reshape(npairs, 1, kgn, 1)
        mu = ref["mean"].reshape(npairs, 1, 1, 1)
        var = ref["var"].reshape(npairs, 1, 1, 1)
    tau_z = 1e-5 * acc + 1e-6
    tau_a = sc / 4.0 * tau_z + 3e-7
    tmax = tau_a.max(axis=(2, 3), keepdims=True)
    tau_mu = tmax + 1e-7
    dev = np.abs(a_g - mu)
    tau_v = 2.0 * dev.max(axis=(2, 3), keepdims=True) * tmax + tmax ** 2 + 1e-6 * var + 1e-12
    rstd = 1.0 / np.sqrt(var + eps)
    y = ref["y"].reshape(a_g.shape)
    tau_y = (ga * rstd * (tau_a + tau_mu) + ga * dev * rstd * tau_v / (2.0 * (var + eps))
             + 2e-6 * (1.0 + np.abs(y)))
    return tau_a.reshape(shp), tau_y.reshape(shp)


def assert_chain_close(y_gpu, ref, scale, gamma, eps, kgn, what=""):
    _, tau_y = chain_tols(ref, scale, gamma, eps, kgn)
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - ref["y"])
    bad = ~(err <= tau_y)
    if bad.any():
        i = np.flatnonzero(bad.reshape(-1))[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside the chain bound; max err/tol = "
            f"{np.nanmax(err / tau_y):.3g}; first {i.tolist()} gpu={y_gpu.reshape(-1)[i].tolist()} "
            f"ref={ref['y'].reshape(-1)[i].tolist()}")
    return float(np.max(err / tau_y))
