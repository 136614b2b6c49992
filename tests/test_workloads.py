"""The seeded input generators both the oracle and the CUDA path draw from:
deterministic per seed, the shapes and distributions the module states, and
the sweep enumerated as documented."""
import math

import pytest
import torch

from direct_convolution_chip_b200 import workloads as wl


def test_named_workloads_are_the_pages_problem_shapes():
    a, b = wl.CONV2D_FULL, wl.CONV1D_FULL
    assert (a.N, a.Cin, a.H, a.W, a.Cout, a.P) == (128, 8, 384, 384, 64, 4)
    assert (b.N, b.C, b.T, b.O, b.K, b.stride, b.pad, b.has_bias) == (32, 256, 4096, 512, 9, 1, 4, True)
    assert len({c.name for c in wl.NAMED}) == 4 and len({c.seed for c in wl.NAMED}) == 4


def test_same_seed_same_inputs_other_seed_other_inputs():
    c = wl.CONV2D_SMALL
    x1, w1, b1 = wl.conv2d_inputs(c)
    x2, w2, b2 = wl.conv2d_inputs(c)
    assert torch.equal(x1, x2) and torch.equal(w1, w2) and torch.equal(b1, b2)
    other = wl.Conv2dCase("other", c.N, c.Cin, c.H, c.W, c.Cout, c.P, seed=c.seed + 1)
    assert not torch.equal(wl.conv2d_inputs(other)[0], x1)
    d = wl.CONV1D_SMALL
    first, second = wl.conv1d_inputs(d), wl.conv1d_inputs(d)
    assert all(torch.equal(u, v) for u, v in zip(first, second))


def test_conv2d_shapes_dtypes_and_distributions():
    c = wl.Conv2dCase("dist", 4, 16, 96, 80, 48, 2, seed=11)
    x, w, b = wl.conv2d_inputs(c)
    assert x.shape == (4, 16, 96, 80) and w.shape == (48, 16, 3, 3) and b.shape == (48,)
    assert x.dtype == w.dtype == b.dtype == torch.float32
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    bound = 1.0 / math.sqrt(16 * 9)
    assert w.abs().max().item() <= bound and b.abs().max().item() <= bound
    assert w.abs().max().item() > 0.9 * bound            # uniform over the whole interval
    assert abs(w.mean().item()) < 0.1 * bound


def test_conv2d_adversarial_variants():
    c = wl.Conv2dCase("adv", 2, 8, 40, 40, 16, 4, seed=5)
    x0, w0, b0 = wl.conv2d_inputs(c)
    x1, w1, b1 = wl.conv2d_inputs(c, x_mean=1.0, w_scale=30.0)
    assert torch.allclose(x1, x0 + 1.0) and torch.allclose(w1, w0 * 30.0) and torch.equal(b1, b0)


def test_conv1d_shapes_and_bounds():
    c = wl.Conv1dCase("dist", 3, 64, 1000, 96, 7, 2, 3, seed=9)
    x, dw, pw, bias = wl.conv1d_inputs(c)
    assert x.shape == (3, 64, 1000) and dw.shape == (64, 7) and pw.shape == (96, 64) and bias.shape == (96,)
    assert dw.abs().max().item() <= 1.0 / math.sqrt(7)
    assert pw.abs().max().item() <= 1.0 / math.sqrt(64) and bias.abs().max().item() <= 1.0 / math.sqrt(64)
    nb = wl.Conv1dCase("nobias", 1, 8, 16, 4, 3, 1, 1, seed=1, has_bias=False)
    assert wl.conv1d_inputs(nb)[3] is None


def test_sweep_enumeration():
    cases = wl.sweep_cases()
    assert len(cases) == 48
    assert [c.op for c in cases] == ["conv2d"] * 16 + ["conv1d"] * 32
    assert [c.seed for c in cases] == [4 + (i % 8) for i in range(48)]
    assert len({c.name for c in cases}) == 48
    c2 = cases[:16]
    assert {(c.Cin, c.Cout, c.H, c.P) for c in c2} == {(ci, co, h, p) for ci in (3, 16) for co in (32, 128)
                                                        for h in (130, 509) for p in (2, 4)}
    assert all(c.N == 16 and c.W == c.H for c in c2)
    c1 = cases[16:]
    assert {(c.C, c.O, c.K, c.stride, c.T) for c in c1} == {(C, O, K, s, T) for C in (64, 384) for O in (128, 768)
                                                            for K in (3, 9) for s in (1, 2) for T in (1000, 16384)}
    assert all(c.N == 8 and c.pad == c.K // 2 for c in c1)


@pytest.mark.parametrize("case", [wl.CONV2D_SMALL, wl.CONV1D_SMALL], ids=lambda c: c.name)
def test_draw_order_is_x_then_weights_then_bias(case):
    """One generator, drawn in the stated order: the weights follow the input's
    draws, so re-drawing them after x from a fresh generator reproduces them."""
    g = torch.Generator("cpu").manual_seed(case.seed)
    if case.op == "conv2d":
        x, w, b = wl.conv2d_inputs(case)
        xr = torch.randn(tuple(x.shape), generator=g, dtype=torch.float32)
        wr = (torch.rand(tuple(w.shape), generator=g, dtype=torch.float32) * 2 - 1) / math.sqrt(case.Cin * 9)
        assert torch.equal(xr, x) and torch.allclose(wr, w, rtol=0, atol=1e-7)
    else:
        x, dw, pw, bias = wl.conv1d_inputs(case)
        xr = torch.randn(tuple(x.shape), generator=g, dtype=torch.float32)
        dwr = (torch.rand(tuple(dw.shape), generator=g, dtype=torch.float32) * 2 - 1) / math.sqrt(case.K)
        assert torch.equal(xr, x) and torch.allclose(dwr, dw, rtol=0, atol=1e-7)
