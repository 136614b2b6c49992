"""ctypes binding of the CPU oracle.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library and
its Python binding never import it, and it never imports them.

All functions take fp32 numpy arrays (C-contiguous) and return float64 numpy
arrays; the arithmetic is the plain double-precision definition in
``fcv_oracle.c``.
"""
import ctypes
import os

import numpy as np

from .build import LIB, build

_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_ip = ctypes.POINTER(ctypes.c_int)


def load(path: str = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(LIB))
    return _lib


def _declare(lib):
    i = ctypes.c_int
    lib.fcvref_num_threads.restype = i
    lib.fcvref_num_threads.argtypes = []
    lib.fcvref_conv2d_out_dims.restype = i
    lib.fcvref_conv2d_out_dims.argtypes = [i, i, i, _ip, _ip, _ip, _ip]
    lib.fcvref_conv1d_out_len.restype = i
    lib.fcvref_conv1d_out_len.argtypes = [i, i, i, i, _ip]
    a2 = [_f32p, _f32p, _f32p, i, i, i, i, i, i]
    lib.fcvref_conv2d_pool_tap.restype = i
    lib.fcvref_conv2d_pool_tap.argtypes = a2 + [_f64p]
    lib.fcvref_conv2d_pool_sigmoid_sum.restype = i
    lib.fcvref_conv2d_pool_sigmoid_sum.argtypes = a2 + [_f64p]
    lib.fcvref_conv2d_pool_tap_at.restype = i
    lib.fcvref_conv2d_pool_tap_at.argtypes = a2 + [_i64p, ctypes.c_int64, _f64p]
    a1 = [_f32p, _f32p, _f32p, _f32p, i, i, i, i, i, i, i]
    lib.fcvref_dwsep_conv1d.restype = i
    lib.fcvref_dwsep_conv1d.argtypes = a1 + [_f64p]
    lib.fcvref_dwsep_conv1d_at.restype = i
    lib.fcvref_dwsep_conv1d_at.argtypes = a1 + [_i64p, ctypes.c_int64, _f64p]
    return lib


def _f32(a):
    a = np.ascontiguousarray(np.asarray(a), dtype=np.float32)
    return a, a.ctypes.data_as(_f32p)


def _opt_f32(a):
    if a is None:
        return None, None
    return _f32(a)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: sizes outside the operation's domain")


def num_threads(lib=None) -> int:
    return (lib or load()).fcvref_num_threads()


def conv2d_out_dims(H, W, P, lib=None):
    """(Ho, Wo, PH, PW) of Conv2d(3x3, s1, p0) then AvgPool2d(P) floor."""
    v = [ctypes.c_int() for _ in range(4)]
    _check((lib or load()).fcvref_conv2d_out_dims(H, W, P, *[ctypes.byref(t) for t in v]),
           "conv2d_out_dims")
    return tuple(t.value for t in v)


def conv1d_out_len(T, K, s, p, lib=None) -> int:
    v = ctypes.c_int()
    _check((lib or load()).fcvref_conv1d_out_len(T, K, s, p, ctypes.byref(v)), "conv1d_out_len")
    return v.value


def _conv2d_dims(x, w, b):
    N, Cin, H, W = x.shape
    Cout = w.shape[0]
    assert w.shape == (Cout, Cin, 3, 3) and b.shape == (Cout,)
    return N, Cin, H, W, Cout


def conv2d_pool_tap(x, w, b, P, lib=None):
    """Pre-sigmoid pooled values, shape [N, Cout, PH, PW], float64."""
    lib = lib or load()
    N, Cin, H, W, Cout = _conv2d_dims(x, w, b)
    _, _, PH, PW = conv2d_out_dims(H, W, P, lib)
    x, xp = _f32(x); w, wp = _f32(w); b, bp = _f32(b)
    out = np.zeros((N, Cout, PH, PW), dtype=np.float64)
    _check(lib.fcvref_conv2d_pool_tap(xp, wp, bp, N, Cin, H, W, Cout, P,
                                      out.ctypes.data_as(_f64p)), "conv2d_pool_tap")
    return out


def conv2d_pool_sigmoid_sum(x, w, b, P, lib=None):
    """out[N] = sum over (C, PH, PW) of sigmoid(avgpool(conv(x))), float64."""
    lib = lib or load()
    N, Cin, H, W, Cout = _conv2d_dims(x, w, b)
    x, xp = _f32(x); w, wp = _f32(w); b, bp = _f32(b)
    out = np.zeros((N,), dtype=np.float64)
    _check(lib.fcvref_conv2d_pool_sigmoid_sum(xp, wp, bp, N, Cin, H, W, Cout, P,
                                              out.ctypes.data_as(_f64p)), "conv2d_pool_sigmoid_sum")
    return out


def conv2d_pool_tap_at(x, w, b, P, idx, lib=None):
    """Pooled pre-sigmoid values at idx[n, 4] = (b, c, ph, pw), float64."""
    lib = lib or load()
    N, Cin, H, W, Cout = _conv2d_dims(x, w, b)
    x, xp = _f32(x); w, wp = _f32(w); b, bp = _f32(b)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 4)
    vals = np.zeros((idx.shape[0],), dtype=np.float64)
    _check(lib.fcvref_conv2d_pool_tap_at(xp, wp, bp, N, Cin, H, W, Cout, P,
                                         idx.ctypes.data_as(_i64p), idx.shape[0],
                                         vals.ctypes.data_as(_f64p)), "conv2d_pool_tap_at")
    return vals


def _conv1d_dims(x, dw, pw, bias):
    N, C, T = x.shape
    O = pw.shape[0]
    K = dw.shape[-1]
    assert dw.reshape(-1).shape[0] == C * K and pw.reshape(O, -1).shape[1] == C
    if bias is not None:
        assert bias.shape == (O,)
    return N, C, T, O, K


def dwsep_conv1d(x, dw, pw, bias, stride, pad, lib=None):
    """Two-stage definition, out[N, O, To] float64.  bias may be None."""
    lib = lib or load()
    N, C, T, O, K = _conv1d_dims(x, dw, pw, bias)
    To = conv1d_out_len(T, K, stride, pad, lib)
    x, xp = _f32(x); dw, dwp = _f32(dw); pw, pwp = _f32(pw); bias, bp = _opt_f32(bias)
    out = np.zeros((N, O, To), dtype=np.float64)
    _check(lib.fcvref_dwsep_conv1d(xp, dwp, pwp, bp, N, C, T, O, K, stride, pad,
                                   out.ctypes.data_as(_f64p)), "dwsep_conv1d")
    return out


def dwsep_conv1d_at(x, dw, pw, bias, stride, pad, idx, lib=None):
    """Outputs at idx[n, 3] = (b, o, t), fused order, float64."""
    lib = lib or load()
    N, C, T, O, K = _conv1d_dims(x, dw, pw, bias)
    x, xp = _f32(x); dw, dwp = _f32(dw); pw, pwp = _f32(pw); bias, bp = _opt_f32(bias)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 3)
    vals = np.zeros((idx.shape[0],), dtype=np.float64)
    _check(lib.fcvref_dwsep_conv1d_at(xp, dwp, pwp, bp, N, C, T, O, K, stride, pad,
                                      idx.ctypes.data_as(_i64p), idx.shape[0],
                                      vals.ctypes.data_as(_f64p)), "dwsep_conv1d_at")
    return vals


__all__ = [
    "load", "build", "num_threads", "conv2d_out_dims", "conv1d_out_len",
    "conv2d_pool_tap", "conv2d_pool_sigmoid_sum", "conv2d_pool_tap_at",
    "dwsep_conv1d", "dwsep_conv1d_at",
]
