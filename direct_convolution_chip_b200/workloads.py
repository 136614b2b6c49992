"""Seeded synthetic workloads for the two fused convolution ops.

This module only draws random inputs.  It holds none of either operation's
arithmetic, so both the CUDA path (through tests and the benchmark) and the CPU
oracle can take their inputs from it.

Shapes are the ones the two POPCORNBENCH traces work on (l2_p65: x[128,8,384,384]
into Conv2d(8->64, 3) and AvgPool2d(4); l2_p7: x[32,256,4096], depthwise K=9,
pointwise 256->512, stride 1, padding 4), plus small and odd-shaped variants.

Distributions: x ~ N(0, 1); every weight and bias ~ U(-1/sqrt(fan_in), +1/sqrt(fan_in))
with fan_in = Cin*9 for the conv2d weight and bias, K for the depthwise weight,
and C for the pointwise weight and bias.  One ``torch.Generator('cpu')`` seeded
with the case's seed draws, in this order: x, then the weights, then the bias.
"""
from dataclasses import dataclass, field
import itertools
import math

import torch


@dataclass(frozen=True)
class Conv2dCase:
    """conv2d(3x3, s1, p0) -> AvgPool2d(P) -> sigmoid -> sum, fp32."""
    name: str
    N: int
    Cin: int
    H: int
    W: int
    Cout: int
    P: int
    seed: int
    tags: tuple = field(default=())

    @property
    def op(self):
        return "conv2d"


@dataclass(frozen=True)
class Conv1dCase:
    """depthwise conv1d(K, stride, pad) -> pointwise conv1d(C -> O) + bias, fp32."""
    name: str
    N: int
    C: int
    T: int
    O: int
    K: int
    stride: int
    pad: int
    seed: int
    has_bias: bool = True
    tags: tuple = field(default=())

    @property
    def op(self):
        return "conv1d"


# The four named workloads.
CONV2D_SMALL = Conv2dCase("conv2d_n2_c8_h64_k16_p4", 2, 8, 64, 64, 16, 4, seed=0, tags=("small",))
CONV1D_SMALL = Conv1dCase("dwsep_n4_c32_t512_o64_k9", 4, 32, 512, 64, 9, 1, 4, seed=1, tags=("small",))
CONV2D_FULL = Conv2dCase("conv2d_n128_c8_h384_k64_p4", 128, 8, 384, 384, 64, 4, seed=2, tags=("full",))
CONV1D_FULL = Conv1dCase("dwsep_n32_c256_t4096_o512_k9", 32, 256, 4096, 512, 9, 1, 4, seed=3, tags=("full",))

NAMED = (CONV2D_SMALL, CONV1D_SMALL, CONV2D_FULL, CONV1D_FULL)


def sweep_cases():
    """The 48-point shape sweep: 16 conv2d points then 32 conv1d points.

    conv2d: Cin in {3,16}, Cout in {32,128}, H=W in {130,509}, pool in {2,4},
    batch 16.  conv1d: C in {64,384}, O in {128,768}, K in {3,9}, stride in
    {1,2}, T in {1000,16384}, pad = K//2, batch 8.  Points are enumerated
    lexicographically in that order; point i (0-based over all 48) uses seed
    4 + (i mod 8).
    """
    cases = []
    i = 0
    for Cin, Cout, H, P in itertools.product((3, 16), (32, 128), (130, 509), (2, 4)):
        cases.append(Conv2dCase(f"sweep_conv2d_c{Cin}_k{Cout}_h{H}_p{P}", 16, Cin, H, H, Cout, P,
                                seed=4 + (i % 8), tags=("sweep",)))
        i += 1
    for C, O, K, s, T in itertools.product((64, 384), (128, 768), (3, 9), (1, 2), (1000, 16384)):
        cases.append(Conv1dCase(f"sweep_dwsep_c{C}_o{O}_k{K}_s{s}_t{T}", 8, C, T, O, K, s, K // 2,
                                seed=4 + (i % 8), tags=("sweep",)))
        i += 1
    return cases


def _uniform(gen, shape, bound):
    return (torch.rand(shape, generator=gen, dtype=torch.float32) * 2.0 - 1.0) * bound


def conv2d_inputs(case: Conv2dCase, x_mean: float = 0.0, w_scale: float = 1.0):
    """(x[N,Cin,H,W], w[Cout,Cin,3,3], b[Cout]) as fp32 CPU tensors.

    ``x_mean`` and ``w_scale`` give the adversarial variants (input off zero
    mean, weights scaled up) that push the sigmoid off its linear range.
    """
    g = torch.Generator("cpu").manual_seed(case.seed)
    x = torch.randn((case.N, case.Cin, case.H, case.W), generator=g, dtype=torch.float32)
    if x_mean:
        x += x_mean
    bound = 1.0 / math.sqrt(case.Cin * 9)
    w = _uniform(g, (case.Cout, case.Cin, 3, 3), bound) * w_scale
    b = _uniform(g, (case.Cout,), bound)
    return x, w, b


def conv1d_inputs(case: Conv1dCase):
    """(x[N,C,T], dw[C,K], pw[O,C], bias[O] or None) as fp32 CPU tensors."""
    g = torch.Generator("cpu").manual_seed(case.seed)
    x = torch.randn((case.N, case.C, case.T), generator=g, dtype=torch.float32)
    dw = _uniform(g, (case.C, case.K), 1.0 / math.sqrt(case.K))
    pw = _uniform(g, (case.O, case.C), 1.0 / math.sqrt(case.C))
    bias = _uniform(g, (case.O,), 1.0 / math.sqrt(case.C)) if case.has_bias else None
    return x, dw, pw, bias
