"""FP64 CPU oracle for the FP32 NCHW conv2d forward and the fused
conv -> bias -> scale -> sigmoid -> GroupNorm chain.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module; the library itself never
does, and this module never imports the library.  The arithmetic lives in
``oracle.c`` (plain C, double precision, OpenMP over independent outputs);
this file only compiles it with gcc and marshals numpy arrays.

Sources are cited in ``oracle.c``: the "GroupConv Atlas" page (problem
statement), the POPCORNBENCH "Kimi-K2.6__l2_p21" transcript (Model forward of
the chain, GroupNorm definition) and the POPCORNBENCH "Kimi-K2.6__l1_p62"
transcript (output size and general index map).

Parity status: pinned (tests/test_oracle.py checks every function against
closed forms, invariants, brute force and library routines in float64).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc -O2 -fopenmp)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        i, p, l = ctypes.c_int, ctypes.c_void_p, ctypes.c_long
        lib.oracle_out_extent.restype = l
        lib.oracle_out_extent.argtypes = [l, l, l, l, l]
        geo = [i] * 14
        lib.oracle_conv2d.restype = i
        lib.oracle_conv2d.argtypes = [p, p, p] + geo + [p, p]
        lib.oracle_conv2d_at.restype = i
        lib.oracle_conv2d_at.argtypes = [p, p, p] + geo + [l, p, p, p]
        lib.oracle_chain.restype = i
        lib.oracle_chain.argtypes = ([p, p, p, p, p, i, p, p, ctypes.c_double] + geo
                                     + [l, p, p, p, p, p, p])
        lib.oracle_num_threads.restype = i
        lib.oracle_num_threads.argtypes = []
        lib.oracle_set_num_threads.restype = None
        lib.oracle_set_num_threads.argtypes = [i]
        _lib = lib
        return lib


def _f32(a):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a), dtype=np.float32)
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _pair(v):
    if isinstance(v, (tuple, list)):
        return int(v[0]), int(v[1])
    return int(v), int(v)


def out_extent(n_in: int, k: int, stride: int, pad: int, dil: int) -> int:
    """Output length along one axis, floor((n + 2p - d(k-1) - 1)/s) + 1."""
    return int(_load().oracle_out_extent(n_in, k, stride, pad, dil))


def _geom(x, w, stride, padding, dilation, groups):
    N, C, H, W = x.shape
    K, cpg, R, S = w.shape
    sh, sw = _pair(stride)
    ph, pw = _pair(padding)
    dh, dw = _pair(dilation)
    if cpg * groups != C:
        raise ValueError("weight shape does not match C/groups")
    P = out_extent(H, R, sh, ph, dh)
    Q = out_extent(W, S, sw, pw, dw)
    if P <= 0 or Q <= 0:
        raise ValueError("kernel larger than padded input")
    return (N, C, H, W, K, R, S, sh, sw, ph, pw, dh, dw, groups), (N, K, P, Q)


def conv2d(x, w, bias=None, stride=1, padding=0, dilation=1, groups=1,
           return_absacc=False):
    """Grouped 2D cross-correlation in float64 on float32 inputs.

    Returns y[N,K,P,Q] (float64) and, if asked, sum|w*x| + |bias| per element.
    """
    x, w, bias = _f32(x), _f32(w), _f32(bias)
    geo, oshape = _geom(x, w, stride, padding, dilation, groups)
    y = np.empty(oshape, dtype=np.float64)
    acc = np.empty(oshape, dtype=np.float64) if return_absacc else None
    st = _load().oracle_conv2d(_ptr(x), _ptr(w), _ptr(bias), *geo, _ptr(y), _ptr(acc))
    if st != 0:
        raise ValueError(f"oracle_conv2d rejected the arguments (status {st})")
    return (y, acc) if return_absacc else y


def conv2d_at(x, w, flat_idx, bias=None, stride=1, padding=0, dilation=1, groups=1):
    """The convolution evaluated only at the given flat output indices.

    Returns (values, sum|w*x| + |bias|), both float64 of len(flat_idx)."""
    x, w, bias = _f32(x), _f32(w), _f32(bias)
    geo, _ = _geom(x, w, stride, padding, dilation, groups)
    idx = np.ascontiguousarray(np.asarray(flat_idx, dtype=np.int64))
    y = np.empty(idx.shape[0], dtype=np.float64)
    acc = np.empty(idx.shape[0], dtype=np.float64)
    st = _load().oracle_conv2d_at(_ptr(x), _ptr(w), _ptr(bias), *geo,
                                  idx.shape[0], _ptr(idx), _ptr(y), _ptr(acc))
    if st != 0:
        raise ValueError(f"oracle_conv2d_at rejected the arguments (status {st})")
    return y, acc


def chain(x, w, b_conv, b_extra, scale, gn_groups, gamma, beta, eps=1e-5,
          stride=1, padding=0, dilation=1, groups=1, pairs=None):
    """conv -> + b_conv + b_extra -> * scale -> sigmoid -> GroupNorm, float64.

    With pairs=None every (n, G) group is computed and the arrays come back as
    [N,K,P,Q]; with pairs=[(n, G), ...] only those groups are computed and the
    arrays are [len(pairs), K/gn_groups, P, Q].
    Returns dict(y, a, absacc, mean, var)."""
    x, w = _f32(x), _f32(w)
    b_conv, b_extra = _f32(b_conv), _f32(b_extra)
    scale, gamma, beta = _f32(scale).reshape(-1), _f32(gamma).reshape(-1), _f32(beta).reshape(-1)
    if b_conv is not None:
        b_conv = b_conv.reshape(-1)
    if b_extra is not None:
        b_extra = b_extra.reshape(-1)
    geo, (N, K, P, Q) = _geom(x, w, stride, padding, dilation, groups)
    if gn_groups <= 0 or K % gn_groups:
        raise ValueError("K must be a multiple of gn_groups")
    kg = K // gn_groups
    if pairs is None:
        npairs, pairs_arr = N * gn_groups, None
        shape = (N, K, P, Q)
    else:
        pairs_arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        npairs = pairs_arr.shape[0]
        shape = (npairs, kg, P, Q)
    y = np.empty(shape, dtype=np.float64)
    a = np.empty(shape, dtype=np.float64)
    acc = np.empty(shape, dtype=np.float64)
    mean = np.empty(npairs, dtype=np.float64)
    var = np.empty(npairs, dtype=np.float64)
    st = _load().oracle_chain(_ptr(x), _ptr(w), _ptr(b_conv), _ptr(b_extra), _ptr(scale),
                              int(gn_groups), _ptr(gamma), _ptr(beta), float(eps), *geo,
                              npairs, _ptr(pairs_arr), _ptr(a), _ptr(y), _ptr(acc),
                              _ptr(mean), _ptr(var))
    if st != 0:
        raise ValueError(f"oracle_chain rejected the arguments (status {st})")
    if pairs is None:
        mean = mean.reshape(N, gn_groups)
        var = var.reshape(N, gn_groups)
    return dict(y=y, a=a, absacc=acc, mean=mean, var=var)


def conv2d_affine_clamp(x, w, scale=None, shift=None, lo=-np.inf, hi=np.inf, stride=1, padding=0,
                        dilation=1, groups=1, return_absacc=False):
    """y = min(max(conv(x, w) * scale[k] + shift[k], lo), hi) in float64: the
    depthwise convolution of the MobileNetV2 inverted-residual block with the
    BatchNorm (inference form, folded into scale and shift) and the ReLU6
    that follow it ("GroupConv Atlas", "Fix the experiment").  scale / shift
    None mean 1 / 0.  The convolution is conv2d above; the affine step and the
    clamp are written out here on its float64 result."""
    y, acc = conv2d(x, w, None, stride, padding, dilation, groups, return_absacc=True)
    K = y.shape[1]
    s = np.ones(K) if scale is None else _f32(scale).reshape(-1).astype(np.float64)
    t = np.zeros(K) if shift is None else _f32(shift).reshape(-1).astype(np.float64)
    y = y * s[None, :, None, None] + t[None, :, None, None]
    y = np.minimum(np.maximum(y, float(lo)), float(hi))
    return (y, acc) if return_absacc else y


def num_threads() -> int:
    """OpenMP threads the oracle runs with."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """OpenMP threads for later calls (timing only; results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))
