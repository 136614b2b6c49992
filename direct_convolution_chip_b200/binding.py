"""Thin ctypes binding of ``libfcv.so`` (the C ABI declared in ``include/fcv.h``).

Argument marshalling only: shapes are read from the tensors, device pointers
and the current CUDA stream are handed to the C entry points, and a nonzero
status becomes an exception.  Every arithmetic step runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and a missing library raises.

PyTorch supplies device memory and streams.  Tensors already on the GPU are
used in place (they must be fp32 and contiguous).  CPU tensors are accepted
too: they are copied to the current device (asynchronously when pinned), the
kernel runs, and the result is copied back into `out` when a CPU tensor is
given (pinned for an asynchronous copy), else into a new pinned CPU tensor --
the path an application with host-resident data takes.  A `stream` argument
orders all of it (copies, allocations, kernel) on that stream.  Host-mode
calls wait for their result copy unless wait=False: the returned CPU tensor
is then valid once that stream has passed the copy, so that a caller can
overlap one call's result copy with the next call's input copy on another
stream.
"""
import ctypes
import functools
import inspect
import os

import torch

from . import build as _build

_LIB = None

ALGO_AUTO = 0
CONV2D_DIRECT = 10
CONV2D_POOLFIRST = 11
CONV2D_TC_3XTF32 = 12
CONV2D_TC_SHIFT_3XTF32 = 13
CONV1D_FMA = 20
CONV1D_TC_3XTF32 = 21
CONV1D_TC2_3XTF32 = 22
CONV1D_TC_TMA_3XTF32 = 23

STATUS_NAMES = {0: "FCV_OK", 1: "FCV_ERR_INVALID_ARG", 2: "FCV_ERR_UNSUPPORTED",
                3: "FCV_ERR_CUDA", 4: "FCV_ERR_TIMEOUT"}

# Every function the header declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
SIGNATURES = {
    "fcv_conv2d_pool_sigmoid_sum": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]),
    "fcv_conv2d_pool_sigmoid_sum_ex": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P]),
    "fcv_conv2d_pool_tap": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P]),
    "fcv_conv2d_pool_sigmoid_sum_det": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, ctypes.c_size_t, _P]),
    "fcv_conv2d_workspace_bytes": (_I, [_I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "fcv_conv2d_pool_sigmoid_sum_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]),
    "fcv_dwsep_conv1d": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "fcv_dwsep_conv1d_ex": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P]),
    "fcv_conv2d_auto_algo": (_I, [_I, _I, _I, _I, _I, _I, ctypes.POINTER(_I)]),
    "fcv_conv2d_tc_plan": (_I, [_I, _I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I),
                                ctypes.POINTER(ctypes.c_uint)]),
    "fcv_dwsep_conv1d_auto_algo": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_I)]),
    "fcv_status_string": (ctypes.c_char_p, [_I]),
    "fcv_version": (_I, []),
    "fcv_device_error": (_I, [_P]),
    "fcv_selftest_wait_timeout": (_I, [ctypes.c_ulonglong, _P]),
    "fcv_selftest_conv2d_stall": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _I, ctypes.c_ulonglong, _P]),
    "fcv_selftest_conv1d_stall": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _I, ctypes.c_ulonglong,
                                       _P]),
    "fcv_selftest_conv1d_pair_stall": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I,
                                            ctypes.c_ulonglong, _P]),
}


class FcvError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def lib_path() -> str:
    return _build.LIB


def load(path: str = None):
    """Load libfcv.so.  Raises if it has not been built: there is no fallback."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or _build.LIB
    if not os.path.exists(p):
        raise RuntimeError(f"libfcv.so not found at {p}: build it with "
                           "`python -m direct_convolution_chip_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _LIB = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load().fcv_status_string(int(status)).decode()
    except RuntimeError:
        return STATUS_NAMES.get(int(status), f"status {status}")


def version() -> int:
    return load().fcv_version()


def _on_stream(fn):
    """Run a binding call with its `stream` argument (when given) as torch's
    current stream, so that everything the call enqueues -- the copies of CPU
    inputs to the device, the buffers it allocates (the caching allocator ties
    them to that stream) and the kernel -- is ordered on that one stream."""
    pos = list(inspect.signature(fn).parameters).index("stream")

    @functools.wraps(fn)
    def call(*args, **kw):
        stream = kw.get("stream", args[pos] if len(args) > pos else None)
        if stream is None:
            return fn(*args, **kw)
        with torch.cuda.stream(stream):
            return fn(*args, **kw)

    return call


def _stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name, device):
    if t is None:
        return None
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32, got {t.dtype}")
    if t.is_cuda:
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return t
    return t.contiguous().to(device, non_blocking=True)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(status, what):
    if status != 0:
        raise FcvError(status, what)


def _host_mode(*ts):
    ts = [t for t in ts if t is not None]
    on_cuda = [t.is_cuda for t in ts]
    if all(on_cuda):
        return False
    if any(on_cuda):
        raise ValueError("pass all tensors on the GPU, or all on the CPU")
    return True


def _result(out_dev, host, stream, out_host=None, wait=True):
    """Host mode: copy the device result into `out_host` (a caller's CPU tensor,
    best pinned) or into a new pinned tensor, and wait for the copy -- or, with
    wait=False, return at once: the CPU tensor then holds the result once the
    stream has reached the end of the copy (e.g. after stream.synchronize())."""
    if not host:
        return out_dev
    if out_host is not None:
        if tuple(out_host.shape) != tuple(out_dev.shape) or out_host.dtype != out_dev.dtype or \
                not out_host.is_contiguous():
            raise ValueError(f"out must be a contiguous {out_dev.dtype} tensor of shape {tuple(out_dev.shape)}")
        res = out_host
    else:
        res = torch.empty(out_dev.shape, dtype=out_dev.dtype, pin_memory=True)
    s = stream or torch.cuda.current_stream()
    with torch.cuda.stream(s):
        res.copy_(out_dev, non_blocking=True)
    if wait:
        s.synchronize()
    return res


def conv2d_out_shape(H, W, pool):
    """(PH, PW) of conv3x3 (stride 1, no padding) followed by AvgPool2d(pool) floor."""
    return (H - 2) // pool, (W - 2) // pool


@_on_stream
def conv2d_pool_sigmoid_sum(x, w, b, pool, out=None, algo=ALGO_AUTO, stream=None, wait=True):
    """out[N] = sum over (C, PH, PW) of sigmoid(avgpool_pool(conv3x3(x, w) + b))."""
    lib = load()
    host = _host_mode(x, w, b)
    dev = torch.device("cuda", torch.cuda.current_device())
    N, Cin, H, W = x.shape
    Cout = w.shape[0]
    if tuple(w.shape) != (Cout, Cin, 3, 3) or tuple(b.shape) != (Cout,):
        raise ValueError(f"w must be [Cout,{Cin},3,3] and b [Cout]; got {tuple(w.shape)}, {tuple(b.shape)}")
    xd, wd, bd = _dev(x, "x", dev), _dev(w, "w", dev), _dev(b, "b", dev)
    out_host = out if host else None
    if out is None or host:
        out = torch.empty((N,), dtype=torch.float32, device=xd.device)
    _check(lib.fcv_conv2d_pool_sigmoid_sum_ex(_ptr(xd), _ptr(wd), _ptr(bd), N, Cin, H, W, Cout, pool,
                                              _ptr(out), algo, _stream_ptr(stream)),
           "fcv_conv2d_pool_sigmoid_sum")
    return _result(out, host, stream, out_host, wait)


def conv2d_workspace_bytes(N, Cin, H, W, Cout, pool) -> int:
    """Workspace bytes the deterministic conv2d sum needs for these sizes."""
    v = ctypes.c_size_t()
    _check(load().fcv_conv2d_workspace_bytes(N, Cin, H, W, Cout, pool, ctypes.byref(v)),
           "fcv_conv2d_workspace_bytes")
    return v.value


@_on_stream
def conv2d_pool_sigmoid_sum_det(x, w, b, pool, out=None, workspace=None, stream=None, wait=True):
    """Bitwise-reproducible variant of conv2d_pool_sigmoid_sum.

    `workspace` is a device tensor of at least conv2d_workspace_bytes(...) bytes
    (allocated here through torch when omitted)."""
    lib = load()
    host = _host_mode(x, w, b)
    dev = torch.device("cuda", torch.cuda.current_device())
    N, Cin, H, W = x.shape
    Cout = w.shape[0]
    if tuple(w.shape) != (Cout, Cin, 3, 3) or tuple(b.shape) != (Cout,):
        raise ValueError("w must be [Cout,Cin,3,3] and b [Cout]")
    need = conv2d_workspace_bytes(N, Cin, H, W, Cout, pool)
    if workspace is None:
        workspace = torch.empty(((need + 15) // 16 * 4,), dtype=torch.float32, device=dev)
    nbytes = workspace.numel() * workspace.element_size()
    xd, wd, bd = _dev(x, "x", dev), _dev(w, "w", dev), _dev(b, "b", dev)
    out_host = out if host else None
    if out is None or host:
        out = torch.empty((N,), dtype=torch.float32, device=xd.device)
    _check(lib.fcv_conv2d_pool_sigmoid_sum_det(_ptr(xd), _ptr(wd), _ptr(bd), N, Cin, H, W, Cout, pool, _ptr(out),
                                               _ptr(workspace) if need else None, nbytes, _stream_ptr(stream)),
           "fcv_conv2d_pool_sigmoid_sum_det")
    return _result(out, host, stream, out_host, wait)


@_on_stream
def conv2d_pool_tap(x, w, b, pool, out=None, algo=ALGO_AUTO, stream=None, wait=True):
    """Pooled pre-sigmoid values [N, Cout, PH, PW] of the same fused kernel."""
    lib = load()
    host = _host_mode(x, w, b)
    dev = torch.device("cuda", torch.cuda.current_device())
    N, Cin, H, W = x.shape
    Cout = w.shape[0]
    if tuple(w.shape) != (Cout, Cin, 3, 3) or tuple(b.shape) != (Cout,):
        raise ValueError("w must be [Cout,Cin,3,3] and b [Cout]")
    PH, PW = conv2d_out_shape(H, W, pool)
    xd, wd, bd = _dev(x, "x", dev), _dev(w, "w", dev), _dev(b, "b", dev)
    out_host = out if host else None
    if out is None or host:
        out = torch.empty((N, Cout, max(PH, 0), max(PW, 0)), dtype=torch.float32, device=xd.device)
    _check(lib.fcv_conv2d_pool_tap(_ptr(xd), _ptr(wd), _ptr(bd), N, Cin, H, W, Cout, pool,
                                   _ptr(out), algo, _stream_ptr(stream)), "fcv_conv2d_pool_tap")
    return _result(out, host, stream, out_host, wait)


def conv1d_out_len(T, K, stride, pad):
    """floor((T + 2*pad - K) / stride) + 1."""
    return (T + 2 * pad - K) // stride + 1


@_on_stream
def dwsep_conv1d(x, dw, pw, bias, stride, pad, out=None, algo=ALGO_AUTO, stream=None, wait=True):
    """out[N, O, To] = pointwise(depthwise(x)) + bias; bias may be None."""
    lib = load()
    host = _host_mode(x, dw, pw, bias)
    dev = torch.device("cuda", torch.cuda.current_device())
    N, C, T = x.shape
    O = pw.shape[0]
    K = dw.shape[-1]
    if dw.numel() != C * K or pw.numel() != O * C or (bias is not None and tuple(bias.shape) != (O,)):
        raise ValueError("dw must be [C,K] (or [C,1,K]), pw [O,C] (or [O,C,1]), bias [O]")
    To = conv1d_out_len(T, K, stride, pad)
    xd, dwd, pwd = _dev(x, "x", dev), _dev(dw, "dw", dev), _dev(pw, "pw", dev)
    bd = _dev(bias, "bias", dev)
    out_host = out if host else None
    if out is None or host:
        out = torch.empty((N, O, max(To, 0)), dtype=torch.float32, device=xd.device)
    _check(lib.fcv_dwsep_conv1d_ex(_ptr(xd), _ptr(dwd), _ptr(pwd), _ptr(bd), N, C, T, O, K, stride, pad,
                                   _ptr(out), algo, _stream_ptr(stream)), "fcv_dwsep_conv1d")
    return _result(out, host, stream, out_host, wait)


def conv2d_tc_plan(Cin, Cout, pool, use_tma=True) -> dict:
    """Diagnostic: what one launch of the tensor-core conv2d uses for these sizes."""
    v, n, t, sm = _I(), _I(), _I(), ctypes.c_uint()
    _check(load().fcv_conv2d_tc_plan(Cin, Cout, pool, int(bool(use_tma)), ctypes.byref(v), ctypes.byref(n),
                                     ctypes.byref(t), ctypes.byref(sm)), "fcv_conv2d_tc_plan")
    return {"variant": "sub-chunk" if v.value else "full-chunk", "nacc": n.value, "tmem_cols": t.value,
            "smem_bytes": sm.value}


def conv2d_auto_algo(N, Cin, H, W, Cout, pool) -> int:
    """The algorithm FCV_ALGO_AUTO runs for these op A sizes (no GPU needed)."""
    a = ctypes.c_int()
    _check(load().fcv_conv2d_auto_algo(N, Cin, H, W, Cout, pool, ctypes.byref(a)), "fcv_conv2d_auto_algo")
    return a.value


def dwsep_conv1d_auto_algo(x, dw, pw, stride, pad) -> int:
    """The algorithm FCV_ALGO_AUTO runs for these op B tensors (only their shapes
    and the 16-byte alignment of x and pw matter; no data is read)."""
    N, C, T = x.shape
    O, K = pw.shape[0], dw.shape[-1]
    a = ctypes.c_int()
    _check(load().fcv_dwsep_conv1d_auto_algo(_ptr(x), _ptr(pw), N, C, T, O, K, stride, pad, ctypes.byref(a)),
           "fcv_dwsep_conv1d_auto_algo")
    return a.value


def device_error(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device error word."""
    return load().fcv_device_error(_stream_ptr(stream))
