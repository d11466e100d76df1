"""FP32 NCHW grouped / depthwise / dense conv2d forward and the fused
conv -> bias -> scale -> sigmoid -> GroupNorm chain on NVIDIA B200 (sm_100a).

This package is a thin binding over the C ABI of ``libgconv.so`` (declared in
include/gconv.h).  It only marshals arguments: every step of the computation
runs in the library's CUDA kernels.  PyTorch supplies device memory and the
current stream.  There is no CPU path: if the library has not been built, or
the tensors are not contiguous FP32 CUDA tensors, calls raise.

Build the library with ``python -m depthwise_convolution_fp32_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "GconvError", "conv2d", "conv2d_affine_clamp", "conv2d_bias_scale_sigmoid_groupnorm", "output_size",
    "plan_name", "force_kernel", "reserve_workspace", "chain_workspace_size",
    "library", "library_path", "status_string", "version",
    "OK", "ERR_INVALID_ARG", "ERR_UNSUPPORTED", "ERR_CUDA", "ERR_WORKSPACE", "ERR_TIMEOUT",
]

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_TIMEOUT = range(6)

_PKG = os.path.dirname(os.path.abspath(__file__))
# GCONV_LIBRARY may point at another build of the same library (A/B measurements).
_LIB_PATH = os.environ.get("GCONV_LIBRARY") or os.path.join(_PKG, "libgconv.so")
_lock = threading.Lock()
_lib = None


class GconvError(RuntimeError):
    """A libgconv entry point returned a non-OK status."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(status)}")


def library_path() -> str:
    return _LIB_PATH


def library():
    """Load libgconv.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"libgconv.so not found at {_LIB_PATH}; build it with "
                "`python -m depthwise_convolution_fp32_b200.build` (there is no CPU fallback)")
        lib = ctypes.CDLL(_LIB_PATH)
        i, p, f, sz, s = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t, ctypes.c_char_p
        geo = [i] * 11
        lib.gconv_status_string.restype = s
        lib.gconv_status_string.argtypes = [i]
        lib.gconv_version.restype = s
        lib.gconv_version.argtypes = []
        lib.gconv2d_output_size.restype = i
        lib.gconv2d_output_size.argtypes = [i] * 7 + [ctypes.POINTER(i), ctypes.POINTER(i)]
        lib.gconv2d_fwd.restype = i
        lib.gconv2d_fwd.argtypes = [p, p, p] + geo + [p, p]
        lib.gconv2d_fwd_ex.restype = i
        lib.gconv2d_fwd_ex.argtypes = [p, p, p] + [i] * 14 + [p, p]
        lib.gconv2d_plan_name_ex.restype = s
        lib.gconv2d_plan_name_ex.argtypes = [i] * 14
        lib.gconv2d_affine_clamp_fwd.restype = i
        lib.gconv2d_affine_clamp_fwd.argtypes = [p, p] + geo + [p, p, f, f, p, p]
        lib.gconv2d_bias_scale_sigmoid_groupnorm_fwd.restype = i
        lib.gconv2d_bias_scale_sigmoid_groupnorm_fwd.argtypes = [p, p, p] + geo + [p, i, p, p, f, p, p]
        lib.gconv2d_chain_workspace_size.restype = sz
        lib.gconv2d_chain_workspace_size.argtypes = geo + [i]
        lib.gconv_reserve_workspace.restype = i
        lib.gconv_reserve_workspace.argtypes = [sz]
        lib.gconv2d_plan_name.restype = s
        lib.gconv2d_plan_name.argtypes = geo + [i]
        lib.gconv_force_kernel.restype = i
        lib.gconv_force_kernel.argtypes = [s]
        lib.gconv_device_error_status.restype = i
        lib.gconv_device_error_status.argtypes = []
        lib.gconv_get_last_device_error.restype = i
        lib.gconv_get_last_device_error.argtypes = [p]
        lib.gconv_selftest_wait_timeout.restype = i
        lib.gconv_selftest_wait_timeout.argtypes = [ctypes.c_uint, p]
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return library().gconv_status_string(int(status)).decode()


def version() -> str:
    return library().gconv_version().decode()


def _check(status: int, where: str):
    if status != OK:
        raise GconvError(status, where)


def output_size(H, W, R, S, stride=1, pad=0, dilation=1):
    P, Q = ctypes.c_int(0), ctypes.c_int(0)
    _check(library().gconv2d_output_size(H, W, R, S, stride, pad, dilation,
                                         ctypes.byref(P), ctypes.byref(Q)), "gconv2d_output_size")
    return P.value, Q.value


def plan_name(N, C, H, W, K, R, S, stride=1, pad=0, dilation=1, groups=1, chain=False) -> str:
    (sh, sw), (ph, pw), (dh, dw) = _pair(stride, "stride"), _pair(pad, "pad"), _pair(dilation, "dilation")
    if sh == sw and ph == pw and dh == dw:
        return library().gconv2d_plan_name(N, C, H, W, K, R, S, sh, ph, dh, groups, 1 if chain else 0).decode()
    if chain:
        raise ValueError("the fused chain takes the same stride, padding and dilation on both axes")
    return library().gconv2d_plan_name_ex(N, C, H, W, K, R, S, sh, sw, ph, pw, dh, dw, groups).decode()


def force_kernel(name: str):
    _check(library().gconv_force_kernel(name.encode()), "gconv_force_kernel")


def reserve_workspace(nbytes: int):
    _check(library().gconv_reserve_workspace(int(nbytes)), "gconv_reserve_workspace")


def chain_workspace_size(N, C, H, W, K, R, S, stride, pad, dilation, groups, gn_groups) -> int:
    return int(library().gconv2d_chain_workspace_size(N, C, H, W, K, R, S, stride, pad, dilation,
                                                      groups, gn_groups))


_torch_mod = None
_SIZES: dict = {}


def _torch():
    global _torch_mod
    if _torch_mod is None:
        import torch
        _torch_mod = torch
    return _torch_mod


_F32 = None


def _dev(t, name, allow_none=False):
    global _F32
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if _F32 is None:
        _F32 = _torch().float32
    try:
        ok = t.is_cuda and t.dtype is _F32 and t.is_contiguous()
    except AttributeError:
        raise TypeError(f"{name} must be a torch.Tensor") from None
    if not ok:
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor "
                         f"(got device={t.device}, dtype={t.dtype}, contiguous={t.is_contiguous()})")
    return t.data_ptr()


_RAW_STREAM = None


def _stream(t):
    """The raw handle of the current stream on t's device."""
    global _RAW_STREAM
    if _RAW_STREAM is None:
        torch = _torch()
        _RAW_STREAM = getattr(torch._C, "_cuda_getCurrentRawStream", None) or \
            (lambda d: torch.cuda.current_stream(d).cuda_stream)
    return _RAW_STREAM(t.get_device())


def _pair(v, name):
    """(h, w) of an int or a 2-tuple argument."""
    if isinstance(v, (tuple, list)):
        if len(v) != 2:
            raise ValueError(f"{name} must be an int or an (h, w) pair")
        return int(v[0]), int(v[1])
    return int(v), int(v)


def _scalar(v, name):
    if isinstance(v, (tuple, list)):
        if len(v) != 2 or v[0] != v[1]:
            raise ValueError(f"{name} must be the same along H and W")
        v = v[0]
    return int(v)


def _out_size(H, W, R, S, stride, padding, dilation):
    key = (H, W, R, S, stride, padding, dilation)
    pq = _SIZES.get(key)
    if pq is None:
        pq = output_size(H, W, R, S, stride, padding, dilation)
        if len(_SIZES) > 4096:
            _SIZES.clear()
        _SIZES[key] = pq
    return pq


def _output(x, out, shape):
    if out is None:
        if x.dtype is not _torch().float32:
            raise ValueError("x must be a contiguous float32 CUDA tensor")
        return x.new_empty(shape)
    if tuple(out.shape) != shape:
        raise ValueError(f"out must have shape {shape}")
    return out


_FWD = None


def conv2d(x, w, bias=None, stride=1, padding=0, dilation=1, groups=1, out=None):
    """y = conv2d(x, w) (+ bias) on the GPU; x[N,C,H,W], w[K,C/groups,R,S].
    stride, padding and dilation are ints or (h, w) pairs."""
    global _FWD
    N, C, H, W = x.shape
    K, cpg, R, S = w.shape
    if type(stride) is int and type(padding) is int and type(dilation) is int:
        sh = sw = stride
        ph = pw = padding
        dh = dw = dilation
    else:
        (sh, sw), (ph, pw), (dh, dw) = _pair(stride, "stride"), _pair(padding, "padding"), _pair(dilation, "dilation")
    if cpg * groups != C:
        raise ValueError("w.shape[1] * groups must equal C")
    if sh == sw and ph == pw and dh == dw:
        P, Q = _out_size(H, W, R, S, sh, ph, dh)
        out = _output(x, out, (N, K, P, Q))
        if _FWD is None:
            _FWD = library().gconv2d_fwd
        st = _FWD(_dev(x, "x"), _dev(w, "w"), _dev(bias, "bias", True),
                  N, C, H, W, K, R, S, sh, ph, dh, groups, _dev(out, "out"), _stream(x))
        if st:
            _check(st, "gconv2d_fwd")
        return out
    P = _out_size(H, H, R, R, sh, ph, dh)[0]
    Q = _out_size(W, W, S, S, sw, pw, dw)[0]
    out = _output(x, out, (N, K, P, Q))
    st = library().gconv2d_fwd_ex(_dev(x, "x"), _dev(w, "w"), _dev(bias, "bias", True),
                                  N, C, H, W, K, R, S, sh, sw, ph, pw, dh, dw, groups, _dev(out, "out"), _stream(x))
    if st:
        _check(st, "gconv2d_fwd_ex")
    return out


def conv2d_affine_clamp(x, w, scale=None, shift=None, lo=float("-inf"), hi=float("inf"), stride=1,
                        padding=0, dilation=1, groups=1, out=None):
    """y = clamp(conv2d(x, w) * scale[k] + shift[k], lo, hi) on the GPU (scale /
    shift [K] or None for 1 / 0).  With BatchNorm folded into scale and shift
    and lo=0, hi=6 this is a convolution + BatchNorm + ReLU6 in one kernel."""
    N, C, H, W = x.shape
    K, cpg, R, S = w.shape
    stride, padding, dilation = (_scalar(stride, "stride"), _scalar(padding, "padding"),
                                 _scalar(dilation, "dilation"))
    if cpg * groups != C:
        raise ValueError("w.shape[1] * groups must equal C")
    for name, t in (("scale", scale), ("shift", shift)):
        if t is not None and t.numel() != K:
            raise ValueError(f"{name} must hold K={K} values")
    P, Q = _out_size(H, W, R, S, stride, padding, dilation)
    out = _output(x, out, (N, K, P, Q))
    st = library().gconv2d_affine_clamp_fwd(_dev(x, "x"), _dev(w, "w"),
                                            N, C, H, W, K, R, S, stride, padding, dilation, groups,
                                            _dev(scale, "scale", True), _dev(shift, "shift", True),
                                            float(lo), float(hi), _dev(out, "out"), _stream(x))
    if st:
        _check(st, "gconv2d_affine_clamp_fwd")
    return out


def conv2d_bias_scale_sigmoid_groupnorm(x, w, bias, scale, gn_groups, gamma, beta, eps=1e-5,
                                        stride=1, padding=0, dilation=1, groups=1, out=None):
    """GroupNorm(sigmoid((conv2d(x, w) + bias) * scale)) with affine gamma/beta.

    bias ([K] or None) is the folded conv bias + extra bias; scale, gamma and
    beta are [K] (a [K,1,1] view is accepted)."""
    N, C, H, W = x.shape
    K, cpg, R, S = w.shape
    stride, padding, dilation = (_scalar(stride, "stride"), _scalar(padding, "padding"),
                                 _scalar(dilation, "dilation"))
    if cpg * groups != C:
        raise ValueError("w.shape[1] * groups must equal C")
    P, Q = _out_size(H, W, R, S, stride, padding, dilation)
    for name, t in (("bias", bias), ("scale", scale), ("gamma", gamma), ("beta", beta)):
        if t is not None and t.numel() != K:
            raise ValueError(f"{name} must hold K={K} values")
    out = _output(x, out, (N, K, P, Q))
    st = library().gconv2d_bias_scale_sigmoid_groupnorm_fwd(
        _dev(x, "x"), _dev(w, "w"), _dev(bias, "bias", True),
        N, C, H, W, K, R, S, stride, padding, dilation, groups,
        _dev(scale, "scale"), int(gn_groups), _dev(gamma, "gamma"), _dev(beta, "beta"),
        float(eps), _dev(out, "out"), _stream(x))
    _check(st, "gconv2d_bias_scale_sigmoid_groupnorm_fwd")
    return out
