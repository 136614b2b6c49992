"""The allocation-free entry point, fcv_conv2d_pool_sigmoid_sum_noalloc.

It exists for callers that must not allocate device memory while they run
(a plugin inside an engine that owns every device allocation, a loop that
cannot take the device synchronisation cudaMalloc/cudaFree can cause, a fixed
memory budget): its workspace is a fixed 256 KiB array that lives in the
library's own device memory.  These tests call it through the C ABI and check
it against the workspace-taking entry point, fcv_conv2d_pool_sigmoid_sum_det,
bit for bit on two calls in a row (the shared array keeps the previous call's
contents, so the second call shows the call clears what it must), and against
the CPU oracle.

This file sorts last so that a run stopping at its first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import oracle
from direct_convolution_chip_b200 import binding
from direct_convolution_chip_b200 import build as fcv_build
from direct_convolution_chip_b200 import workloads as wl
from tests.parity import assert_close, requires_cuda

P = ctypes.c_void_p
UNSUPPORTED = 2


@pytest.fixture(scope="module")
def lib():
    fcv_build.build()
    return binding.load()


def _ptr(t):
    return P(t.data_ptr())


def test_rejects_sizes_beyond_the_static_scratch(lib):
    """1024 images of 384x384 at pool 4 need 590 KB of workspace: refused on
    the host, before any CUDA call (no GPU needed)."""
    fake = P(0x10000)
    need = ctypes.c_size_t()
    assert lib.fcv_conv2d_workspace_bytes(1024, 8, 384, 384, 64, 4, ctypes.byref(need)) == 0
    assert need.value > 256 * 1024
    assert lib.fcv_conv2d_pool_sigmoid_sum_noalloc(fake, fake, fake, 1024, 8, 384, 384, 64, 4, fake,
                                                   None) == UNSUPPORTED


@pytest.mark.gpu
@requires_cuda
@pytest.mark.parametrize("case", [wl.CONV2D_SMALL, wl.CONV2D_FULL,
                                  wl.Conv2dCase("noalloc_odd", 3, 5, 61, 47, 70, 3, seed=17)],
                         ids=lambda c: c.name)
def test_noalloc_matches_workspace_entry_point_twice(lib, case):
    x, w, b = [t.cuda() for t in wl.conv2d_inputs(case)]
    stream = P(torch.cuda.current_stream().cuda_stream)
    dims = (case.N, case.Cin, case.H, case.W, case.Cout, case.P)

    need = ctypes.c_size_t()
    assert lib.fcv_conv2d_workspace_bytes(*dims, ctypes.byref(need)) == 0
    assert need.value <= 256 * 1024
    ws = torch.empty(((need.value + 15) // 16 * 4,), dtype=torch.float32, device="cuda")
    ref = torch.empty((case.N,), dtype=torch.float32, device="cuda")
    assert lib.fcv_conv2d_pool_sigmoid_sum_det(_ptr(x), _ptr(w), _ptr(b), *dims, _ptr(ref), _ptr(ws),
                                               need.value, stream) == 0

    results = []
    for _ in range(2):  # two calls in a row share the one static array
        out = torch.full((case.N,), float("nan"), device="cuda")
        assert lib.fcv_conv2d_pool_sigmoid_sum_noalloc(_ptr(x), _ptr(w), _ptr(b), *dims, _ptr(out), stream) == 0
        results.append(out)
    torch.cuda.synchronize()
    assert lib.fcv_device_error(stream) == 0
    # Both entry points run the same kernel and add the partial sums in the
    # same fixed order, so the results agree bit for bit.
    for i, out in enumerate(results):
        assert torch.equal(out, ref), f"{case.name} call {i}: differs from the workspace entry point"
    # ... and they match the CPU oracle on the first and last batch items.
    xn, wn, bn = [t.cpu().numpy() for t in (x, w, b)]
    for bi in sorted({0, case.N - 1}):
        want = oracle.conv2d_pool_sigmoid_sum(xn[bi:bi + 1], wn, bn, case.P)
        assert_close(results[1][bi:bi + 1].cpu().double().numpy(), want, f"{case.name} item {bi} vs oracle")
