"""The failure path of the production tensor-core kernels, on the GPU, without
a fault: one role of every thread block waits on a barrier that nothing
completes, with a short limit (fcv_selftest_conv2d_stall /
fcv_selftest_conv1d_stall / fcv_selftest_conv1d_pair_stall).  The wait must give up and record FCV_ERR_TIMEOUT;
every other role must then leave its loop, the TMA copies and MMAs already in
flight must be waited for and tensor memory freed, so the context stays usable:
the next normal call on the same inputs matches the CPU oracle.

The roles are 1 loader / TMA warp, 2 producers, 3 MMA issuer, 4 epilogue.  A
stall at unit (or tile) 0 hits before any MMA; at 2 it hits with boxes landed,
MMAs committed and an accumulator in the epilogue.  The shapes give every
thread block at least three units, so every block stalls.
"""
import ctypes

import pytest
import torch

import oracle
from direct_convolution_chip_b200 import binding
from direct_convolution_chip_b200 import build as fcv_build
from direct_convolution_chip_b200 import workloads as wl
from tests.parity import assert_close, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]

P = ctypes.c_void_p
TIMEOUT = 4
LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module")
def lib():
    fcv_build.build()
    return binding.load()


def _p(t):
    return P(t.data_ptr())


CONV2D_STALL = [
    wl.Conv2dCase("stall_tma", 32, 8, 132, 132, 64, 4, seed=31),     # W % 4 == 0: TMA rows, 512 units
    wl.Conv2dCase("stall_cp", 32, 16, 130, 130, 70, 2, seed=32),     # cp.async rows, two K chunks, two launches
]


@pytest.mark.parametrize("case", CONV2D_STALL, ids=lambda c: c.name)
def test_conv2d_stall_every_role(lib, case):
    x, w, b = [t.cuda() for t in wl.conv2d_inputs(case)]
    out = torch.empty(case.N, device="cuda")
    sp = P(torch.cuda.current_stream().cuda_stream)
    assert lib.fcv_device_error(sp) == 0
    for role in (1, 2, 3, 4):
        for at in (0, 2):
            st = lib.fcv_selftest_conv2d_stall(_p(x), _p(w), _p(b), case.N, case.Cin, case.H, case.W, case.Cout,
                                               case.P, _p(out), role, at, LIMIT_NS, sp)
            assert st == 0, f"role {role} at {at}: launch status {st}"
            assert lib.fcv_device_error(sp) == TIMEOUT, f"role {role} at {at}: no timeout recorded"
    # the context still works: a normal call matches the oracle
    got = binding.conv2d_pool_sigmoid_sum(x, w, b, case.P, algo=binding.CONV2D_TC_SHIFT_3XTF32)
    tap = binding.conv2d_pool_tap(x, w, b, case.P, algo=binding.CONV2D_TC_SHIFT_3XTF32)
    torch.cuda.synchronize()
    assert lib.fcv_device_error(sp) == 0
    xn, wn, bn = x.cpu().numpy(), w.cpu().numpy(), b.cpu().numpy()
    for bi in (0, case.N - 1):
        assert_close(got[bi:bi + 1], oracle.conv2d_pool_sigmoid_sum(xn[bi:bi + 1], wn, bn, case.P), f"out[{bi}]")
        assert_close(tap[bi:bi + 1], oracle.conv2d_pool_tap(xn[bi:bi + 1], wn, bn, case.P), f"tap[{bi}]")


@pytest.mark.parametrize("stride", [1, 2])
def test_conv1d_stall_every_role(lib, stride):
    # 320 tiles either way: every block has >= 2
    T = 1024 * stride
    case = wl.Conv1dCase("stall", 40, 64, T, 256, 9, stride, 4, seed=33 + stride)
    x, dw, pw, bias = [t.cuda() for t in wl.conv1d_inputs(case)]
    To = binding.conv1d_out_len(case.T, case.K, case.stride, case.pad)
    out = torch.empty((case.N, case.O, To), device="cuda")
    sp = P(torch.cuda.current_stream().cuda_stream)
    assert lib.fcv_device_error(sp) == 0
    for role in (1, 2, 3, 4):
        for at in (0, 1):
            st = lib.fcv_selftest_conv1d_stall(_p(x), _p(dw), _p(pw), _p(bias), case.N, case.C, case.T, case.O,
                                               case.K, case.stride, case.pad, _p(out), role, at, LIMIT_NS, sp)
            assert st == 0, f"role {role} at {at}: launch status {st}"
            assert lib.fcv_device_error(sp) == TIMEOUT, f"role {role} at {at}: no timeout recorded"
    got = binding.dwsep_conv1d(x, dw, pw, bias, case.stride, case.pad, algo=binding.CONV1D_TC_TMA_3XTF32)
    torch.cuda.synchronize()
    assert lib.fcv_device_error(sp) == 0
    xn, dwn, pwn, bn = [t.cpu().numpy() for t in (x, dw, pw, bias)]
    for bi in (0, case.N - 1):
        want = oracle.dwsep_conv1d(xn[bi:bi + 1], dwn, pwn, bn, case.stride, case.pad)
        assert_close(got[bi:bi + 1], want, f"out[{bi}]")


@pytest.mark.parametrize("stride", [1, 2])
def test_conv1d_pair_stall_every_role(lib, stride):
    """The SM-pair kernel: one role of one CTA of every pair stalls; that CTA
    gives up, its peer sees the abort flag through distributed shared memory,
    both drain what is in flight and free tensor memory, and the next normal
    call matches the oracle.  Roles: 1 TMA warp, 2 producers, 3 MMA issuer
    (rank 0 only), 4 epilogue, 5 pw split, 6 relay (rank 1 only)."""
    # 40 x 4 x 2 = 320 pair tiles on 74 pairs: every pair has >= 4
    case = wl.Conv1dCase("pair_stall", 40, 256, 1024 * stride, 512, 9, stride, 4, seed=37 + stride)
    x, dw, pw, bias = [t.cuda() for t in wl.conv1d_inputs(case)]
    To = binding.conv1d_out_len(case.T, case.K, case.stride, case.pad)
    out = torch.empty((case.N, case.O, To), device="cuda")
    sp = P(torch.cuda.current_stream().cuda_stream)
    assert lib.fcv_device_error(sp) == 0
    roles = ((1, (0, 1)), (2, (0, 1)), (3, (0,)), (4, (0, 1)), (5, (0, 1)), (6, (1,)))
    for role, ranks in roles if stride == 1 else [r for r in roles if r[0] != 5]:  # no split warps at stride 2
        for rank in ranks:
            for at in (0, 2):
                st = lib.fcv_selftest_conv1d_pair_stall(_p(x), _p(dw), _p(pw), _p(bias), case.N, case.C, case.T,
                                                        case.O, case.K, case.stride, case.pad, _p(out), role, at,
                                                        rank, LIMIT_NS, sp)
                assert st == 0, f"role {role} rank {rank} at {at}: launch status {st}"
                assert lib.fcv_device_error(sp) == TIMEOUT, f"role {role} rank {rank} at {at}: no timeout recorded"
    got = binding.dwsep_conv1d(x, dw, pw, bias, case.stride, case.pad, algo=binding.CONV1D_TC2_3XTF32)
    torch.cuda.synchronize()
    assert lib.fcv_device_error(sp) == 0
    xn, dwn, pwn, bn = [t.cpu().numpy() for t in (x, dw, pw, bias)]
    for bi in (0, case.N - 1):
        want = oracle.dwsep_conv1d(xn[bi:bi + 1], dwn, pwn, bn, case.stride, case.pad)
        assert_close(got[bi:bi + 1], want, f"out[{bi}]")
