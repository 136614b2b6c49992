"""Fused small-channel direct convolution for NVIDIA B200 (sm_100a).

The kernels live in ``libfcv.so`` behind the C ABI of ``include/fcv.h``;
``binding`` is its thin ctypes wrapper.  Importing this package loads nothing:
the library is loaded on first use and raises if it has not been built.
"""
from .binding import (ALGO_AUTO, CONV1D_FMA, CONV1D_TC2_3XTF32, CONV1D_TC_3XTF32, CONV1D_TC_TMA_3XTF32, CONV2D_DIRECT, CONV2D_POOLFIRST, CONV2D_TC_3XTF32, CONV2D_TC_SHIFT_3XTF32, FcvError,
                      conv1d_out_len, conv2d_auto_algo, conv2d_out_shape, conv2d_tc_plan, conv2d_pool_sigmoid_sum, conv2d_pool_sigmoid_sum_det,
                      conv2d_pool_tap, conv2d_workspace_bytes,
                      device_error, dwsep_conv1d, dwsep_conv1d_auto_algo, load, status_string, version)

__all__ = [
    "ALGO_AUTO", "CONV1D_FMA", "CONV1D_TC2_3XTF32", "CONV1D_TC_3XTF32", "CONV1D_TC_TMA_3XTF32", "CONV2D_DIRECT", "CONV2D_POOLFIRST", "CONV2D_TC_3XTF32", "CONV2D_TC_SHIFT_3XTF32", "FcvError",
    "conv1d_out_len", "conv2d_auto_algo", "conv2d_out_shape", "conv2d_tc_plan", "conv2d_pool_sigmoid_sum", "conv2d_pool_sigmoid_sum_det",
    "conv2d_pool_tap", "conv2d_workspace_bytes",
    "device_error", "dwsep_conv1d", "dwsep_conv1d_auto_algo", "load", "status_string", "version",
]
