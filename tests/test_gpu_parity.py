"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs, element by element at allclose(atol=rtol=1e-4).

Small workloads are compared in full.  The full-size workloads and the shape
sweep are compared on whole batch items the oracle can finish in seconds and
on sampled outputs the oracle evaluates one by one, all produced by the same
entry points (and launch configuration) the benchmark times.
"""
import numpy as np
import pytest
import torch

import direct_convolution_chip_b200 as fcv
import oracle
from direct_convolution_chip_b200 import workloads as wl
from tests.parity import assert_close, requires_cuda, sample_indices

pytestmark = [pytest.mark.gpu, requires_cuda]

CONV2D_ALGOS = [fcv.CONV2D_DIRECT, fcv.CONV2D_POOLFIRST, fcv.CONV2D_TC_3XTF32, fcv.CONV2D_TC_SHIFT_3XTF32]
CONV2D_TC_ALGOS = (fcv.CONV2D_TC_3XTF32, fcv.CONV2D_TC_SHIFT_3XTF32)
CONV1D_ALGOS = [fcv.CONV1D_FMA, fcv.CONV1D_TC_3XTF32, fcv.CONV1D_TC2_3XTF32, fcv.CONV1D_TC_TMA_3XTF32]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from direct_convolution_chip_b200 import build
    build.build()
    fcv.load()


def cuda(*ts):
    return [None if t is None else t.cuda() for t in ts]


def conv1d_or_skip(x, dw, pw, bias, s, p, algo):
    try:
        return fcv.dwsep_conv1d(x, dw, pw, bias, s, p, algo=algo)
    except fcv.FcvError as e:
        if e.status == 2 and algo in (fcv.CONV1D_TC_3XTF32, fcv.CONV1D_TC2_3XTF32, fcv.CONV1D_TC_TMA_3XTF32):
            pytest.skip("tensor-core path does not cover this shape")
        raise


# ------------------------------------------------------------------ op A ---

def conv2d_or_skip(fn, x, w, b, pool, algo):
    try:
        return fn(x, w, b, pool, algo=algo)
    except fcv.FcvError as e:
        if e.status == 2 and algo in CONV2D_TC_ALGOS:
            pytest.skip("this tensor-core conv2d does not cover this shape")
        raise


def check_conv2d_case(case, algo, batch_items=None, n_samples=2000, x_mean=0.0, w_scale=1.0):
    x, w, b = wl.conv2d_inputs(case, x_mean=x_mean, w_scale=w_scale)
    xd, wd, bd = cuda(x, w, b)
    out = conv2d_or_skip(fcv.conv2d_pool_sigmoid_sum, xd, wd, bd, case.P, algo)
    tap = conv2d_or_skip(fcv.conv2d_pool_tap, xd, wd, bd, case.P, algo)
    torch.cuda.synchronize()
    xn, wn, bn = x.numpy(), w.numpy(), b.numpy()
    items = range(case.N) if batch_items is None else batch_items
    for bi in items:
        xs = xn[bi:bi + 1]
        assert_close(out[bi:bi + 1], oracle.conv2d_pool_sigmoid_sum(xs, wn, bn, case.P), f"{case.name} out[{bi}]")
        assert_close(tap[bi:bi + 1], oracle.conv2d_pool_tap(xs, wn, bn, case.P), f"{case.name} tap[{bi}]")
    if n_samples and tap.numel():
        idx = sample_indices(tuple(tap.shape), n_samples, seed=case.seed)
        ref = oracle.conv2d_pool_tap_at(xn, wn, bn, case.P, idx)
        got = tap.cpu().numpy()[idx[:, 0], idx[:, 1], idx[:, 2], idx[:, 3]]
        assert_close(got, ref, f"{case.name} tap samples")
    return out, tap


@pytest.mark.parametrize("algo", CONV2D_ALGOS)
def test_conv2d_small_full(algo):
    check_conv2d_case(wl.CONV2D_SMALL, algo, n_samples=0)


@pytest.mark.parametrize("algo", CONV2D_ALGOS)
def test_conv2d_full_size(algo):
    """x[128,8,384,384], Cout 64, pool 4: items 0, 63, 127 in full, 4096 sampled pooled values."""
    check_conv2d_case(wl.CONV2D_FULL, algo, batch_items=[0, 63, 127], n_samples=4096)


@pytest.mark.parametrize("case", [c for c in wl.sweep_cases() if c.op == "conv2d"], ids=lambda c: c.name)
@pytest.mark.parametrize("algo", CONV2D_ALGOS)
def test_conv2d_sweep(case, algo):
    heavy = case.Cin * case.Cout * case.H * case.W > 16 * 128 * 200 * 200
    check_conv2d_case(case, algo, batch_items=[0] if heavy else [0, case.N - 1], n_samples=2000)


EDGE_2D = [
    # (N, Cin, H, W, Cout, P)
    (1, 1, 3, 3, 1, 1),        # smallest image: one conv output
    (2, 3, 9, 9, 5, 1),
    (1, 2, 11, 13, 7, 3),      # ragged floors in both dims
    (3, 5, 37, 29, 17, 2),     # Cout not a multiple of the channel group
    (1, 4, 41, 70, 33, 5),
    (2, 2, 30, 31, 3, 6),
    (1, 3, 25, 60, 9, 7),
    (1, 2, 44, 50, 4, 8),
    (2, 8, 70, 90, 130, 4),    # more than one channel block
    (1, 20, 35, 36, 6, 4),     # more than one input-channel chunk
    (1, 3, 509, 509, 1, 4),    # single output channel, large odd image
    (4, 1, 130, 3, 2, 1),      # one conv column
    # tensor-core conv2d envelope
    (2, 8, 50, 52, 112, 2),    # the widest Cout: full-chunk kernel, two accumulators, TMA halo
    (1, 24, 40, 44, 48, 4),    # sub-chunk kernel: three input-channel chunks, three accumulators
    (3, 5, 66, 64, 20, 1),     # sub-chunk kernel, pool 1, Cout padded to 32
    (1, 8, 36, 68, 96, 2),     # sub-chunk kernel at its widest Cout: two accumulators, all 512 TMEM columns
    (1, 16, 36, 68, 96, 2),    # weights too large for the tensor-core kernel: AUTO and FMA only
    (2, 8, 48, 40, 80, 8),     # sub-chunk kernel, pool 8, Cout 80 (two accumulators)
    (1, 9, 30, 34, 64, 4),     # W % 4 != 0: full-chunk kernel with the cp.async halo
    # shifted-operand tensor-core conv2d envelope
    (5, 8, 40, 76, 64, 4),     # N % 4 != 0: the last image group is partial (TMA rows)
    (6, 16, 30, 41, 200, 2),   # two K chunks, four launches of <= 64 channels, cp.async rows, N % 4 != 0
    (9, 3, 21, 134, 64, 8),    # Cin padded to 8, pool 8, three column tiles with a ragged last one
    (4, 12, 19, 20, 65, 1),    # pool 1, Cout one past a block, W % 4 == 0 with two K chunks
    (2, 7, 67, 257, 31, 4),    # W % 4 == 1 (every row a different 16-byte phase), ragged tiles
    (1, 16, 10, 10, 1, 2),     # a single unit: the CTA has no continuation
]


@pytest.mark.parametrize("shape", EDGE_2D, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("algo", CONV2D_ALGOS)
def test_conv2d_edges(shape, algo):
    N, Cin, H, W, Cout, P = shape
    case = wl.Conv2dCase("edge", N, Cin, H, W, Cout, P, seed=sum(shape))
    check_conv2d_case(case, algo, n_samples=0)


def test_conv2d_empty_pool_gives_zero():
    """Ho = 3 < pool = 4: PH = 0, so out = 0 (the library zeroes out itself)."""
    case = wl.Conv2dCase("empty", 3, 2, 5, 40, 4, 4, seed=9)
    x, w, b = cuda(*wl.conv2d_inputs(case))
    out = torch.full((3,), 7.0, device="cuda")
    fcv.conv2d_pool_sigmoid_sum(x, w, b, 4, out=out)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    assert fcv.conv2d_pool_tap(x, w, b, 4).numel() == 0


@pytest.mark.parametrize("variant", [dict(w_scale=30.0), dict(x_mean=1.0), dict(x_mean=1.0, w_scale=30.0)],
                         ids=["w_x30", "x_mean1", "both"])
@pytest.mark.parametrize("algo", CONV2D_ALGOS)
def test_conv2d_adversarial(variant, algo):
    """Weights x30 and/or x ~ N(1,1): the sigmoid leaves its linear range."""
    case = wl.Conv2dCase("adv", 2, 8, 96, 80, 24, 4, seed=21)
    check_conv2d_case(case, algo, n_samples=0, **variant)


def test_conv2d_output_fully_overwritten():
    case = wl.CONV2D_SMALL
    x, w, b = cuda(*wl.conv2d_inputs(case))
    ref = fcv.conv2d_pool_sigmoid_sum(x, w, b, case.P).clone()
    out = torch.full_like(ref, 1e30)
    fcv.conv2d_pool_sigmoid_sum(x, w, b, case.P, out=out)
    torch.cuda.synchronize()
    assert torch.allclose(out, ref, rtol=1e-6, atol=0)


# ------------------------------------------------------------------ op B ---

def check_conv1d_case(case, algo, full_items=None, n_samples=2000, bias_none=False):
    x, dw, pw, bias = wl.conv1d_inputs(case)
    if bias_none:
        bias = None
    xd, dwd, pwd, bd = cuda(x, dw, pw, bias)
    out = conv1d_or_skip(xd, dwd, pwd, bd, case.stride, case.pad, algo)
    torch.cuda.synchronize()
    xn, dwn, pwn = x.numpy(), dw.numpy(), pw.numpy()
    bn = None if bias is None else bias.numpy()
    items = range(case.N) if full_items is None else full_items
    for bi in items:
        ref = oracle.dwsep_conv1d(xn[bi:bi + 1], dwn, pwn, bn, case.stride, case.pad)
        assert_close(out[bi:bi + 1], ref, f"{case.name} out[{bi}]")
    if n_samples:
        idx = sample_indices(tuple(out.shape), n_samples, seed=case.seed)
        ref = oracle.dwsep_conv1d_at(xn, dwn, pwn, bn, case.stride, case.pad, idx)
        got = out.cpu().numpy()[idx[:, 0], idx[:, 1], idx[:, 2]]
        assert_close(got, ref, f"{case.name} samples")
    return out


@pytest.mark.parametrize("algo", CONV1D_ALGOS)
def test_conv1d_small_full(algo):
    check_conv1d_case(wl.CONV1D_SMALL, algo, n_samples=0)


@pytest.mark.parametrize("algo", CONV1D_ALGOS)
def test_conv1d_full_size(algo):
    """x[32,256,4096] -> [32,512,4096]: items 0 and 31 in full, 4096 sampled outputs."""
    check_conv1d_case(wl.CONV1D_FULL, algo, full_items=[0, 31], n_samples=4096)


def test_conv1d_auto_matches_oracle():
    check_conv1d_case(wl.CONV1D_SMALL, fcv.ALGO_AUTO, n_samples=0)


@pytest.mark.parametrize("case", [c for c in wl.sweep_cases() if c.op == "conv1d"], ids=lambda c: c.name)
@pytest.mark.parametrize("algo", CONV1D_ALGOS)
def test_conv1d_sweep(case, algo):
    full = [0] if case.T <= 1000 else []
    check_conv1d_case(case, algo, full_items=full, n_samples=2000)


EDGE_1D = [
    # (N, C, T, O, K, s, p, bias)
    (1, 1, 1, 1, 1, 1, 0, True),      # single sample, K = 1
    (2, 3, 17, 5, 3, 1, 1, False),    # no bias
    (1, 7, 130, 9, 9, 2, 4, True),    # stride 2, odd sizes
    (2, 5, 300, 129, 5, 3, 0, True),  # stride 3, no padding, O just over a tile
    (1, 17, 257, 200, 9, 1, 12, True),  # pad larger than K
    (1, 33, 64, 16, 32, 1, 16, True),   # the largest supported K
    (1, 16, 1000, 64, 1, 1, 0, True),   # pointwise only (K = 1)
    (3, 40, 129, 33, 7, 8, 3, False),   # the largest supported stride
    (1, 300, 70, 20, 4, 1, 1, True),    # C not a multiple of the channel chunk
    # TMA-halo tensor-core kernel (T % 4 == 0): every halo offset r = (-pad) mod 4
    (2, 32, 1000, 64, 5, 1, 2, True),   # r = 2
    (2, 36, 512, 48, 7, 1, 3, True),    # r = 1, a partial second channel chunk
    (1, 64, 256, 300, 13, 1, 5, False), # r = 3 with the largest tensor-core K, partial output tile
    (1, 8, 4, 8, 3, 1, 1, True),        # T = 4: one partial time tile
    # the same kernel at stride 2 (the halo in two TMA boxes): every r, ragged tiles
    (2, 32, 1000, 64, 9, 2, 4, True),   # r = 0, K = 9
    (1, 36, 516, 300, 13, 2, 5, False), # r = 3 with the largest tensor-core K, partial output tile
    (3, 17, 260, 33, 3, 2, 1, True),    # r = 3, K = 3, C not a multiple of 4 (register/FMA paths)
    (2, 64, 2048, 256, 5, 2, 2, True),  # r = 2
    (1, 40, 300, 20, 4, 2, 0, True),    # even K, no padding
    (1, 16, 256, 40, 3, 2, 7, True),    # pad larger than K, r = 1
    (1, 8, 4, 8, 3, 2, 1, True),        # T = 4: To = 2
    # where AUTO takes the SM-pair kernel (stride 1, C >= 256, O >= 256): ragged in every dimension
    (2, 260, 1000, 300, 9, 1, 4, True), # 9 channel chunks (the last 4 wide), last pair tile 232 times, O tile 44 wide
    (1, 256, 516, 256, 3, 1, 1, False), # K = 3, r = 3, no bias, last pair tile 4 times
    (3, 288, 4, 512, 9, 1, 4, True),    # T = 4: one 4-time tile per item, fewer tiles than SM pairs
]


@pytest.mark.parametrize("shape", EDGE_1D, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("algo", CONV1D_ALGOS)
def test_conv1d_edges(shape, algo):
    N, C, T, O, K, s, p, has_bias = shape
    case = wl.Conv1dCase("edge", N, C, T, O, K, s, p, seed=sum(shape[:7]), has_bias=has_bias)
    check_conv1d_case(case, algo, n_samples=0)


# ------------------------------------------------------- both ops, hygiene ---

def _guarded(n, fill=float("nan"), guard=1024):
    buf = torch.full((n + 2 * guard,), fill, device="cuda")
    return buf, buf[guard:guard + n]


def test_guard_bands_untouched():
    """Outputs inside NaN-filled guard regions: nothing outside the output is written."""
    guard = 1024
    case = wl.Conv2dCase("canary", 3, 5, 61, 47, 19, 4, seed=5)
    x, w, b = cuda(*wl.conv2d_inputs(case))
    PH, PW = fcv.conv2d_out_shape(case.H, case.W, case.P)
    buf, out = _guarded(case.N)
    fcv.conv2d_pool_sigmoid_sum(x, w, b, case.P, out=out)
    tbuf, tap = _guarded(case.N * case.Cout * PH * PW)
    fcv.conv2d_pool_tap(x, w, b, case.P, out=tap.view(case.N, case.Cout, PH, PW))
    c1 = wl.Conv1dCase("canary", 2, 19, 333, 37, 9, 2, 4, seed=6)
    xs, dw, pw, bias = cuda(*wl.conv1d_inputs(c1))
    To = fcv.conv1d_out_len(c1.T, c1.K, c1.stride, c1.pad)
    results = []
    for algo in CONV1D_ALGOS:
        obuf, o = _guarded(c1.N * c1.O * To)
        try:
            fcv.dwsep_conv1d(xs, dw, pw, bias, c1.stride, c1.pad, out=o.view(c1.N, c1.O, To), algo=algo)
        except fcv.FcvError as e:
            if e.status != 2:
                raise
            continue
        results.append((obuf, o))
    torch.cuda.synchronize()
    for b_, o_ in [(buf, out), (tbuf, tap)] + results:
        assert torch.isnan(b_[:guard]).all() and torch.isnan(b_[-guard:]).all()
        assert torch.isfinite(o_).all()


def _guarded_copy(t, guard=1024):
    """t's values inside a NaN-filled device buffer with `guard` floats on each
    side (4 KiB: the 16-byte alignment the TMA paths need is kept)."""
    buf = torch.full((t.numel() + 2 * guard,), float("nan"), device="cuda")
    view = buf[guard:guard + t.numel()].view(t.shape)
    view.copy_(t)
    return buf, view


def _check_guards_and_inputs(guarded, originals, guard=1024):
    for (buf, view), orig in zip(guarded, originals):
        assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[-guard:]).all(), "a guard region changed"
        assert torch.equal(view, orig), "an input changed"


@pytest.mark.parametrize("W", [48, 47], ids=["tma", "cp_async"])
@pytest.mark.parametrize("algo", CONV2D_ALGOS)
def test_conv2d_inputs_in_guard_regions(algo, W):
    """Every input inside NaN guard regions: a read past an input's ends would
    turn outputs into NaN, so oracle parity shows none happens; the inputs and
    their guards are unchanged afterwards."""
    case = wl.Conv2dCase("inguard", 3, 5, 61, W, 19, 4, seed=7)
    x, w, b = wl.conv2d_inputs(case)
    originals = cuda(x, w, b)
    guarded = [_guarded_copy(t) for t in originals]
    xg, wg, bg = [v for _, v in guarded]
    out = conv2d_or_skip(fcv.conv2d_pool_sigmoid_sum, xg, wg, bg, case.P, algo)
    tap = conv2d_or_skip(fcv.conv2d_pool_tap, xg, wg, bg, case.P, algo)
    torch.cuda.synchronize()
    _check_guards_and_inputs(guarded, originals)
    xn, wn, bn = x.numpy(), w.numpy(), b.numpy()
    assert_close(out, oracle.conv2d_pool_sigmoid_sum(xn, wn, bn, case.P), "out")
    assert_close(tap, oracle.conv2d_pool_tap(xn, wn, bn, case.P), "tap")


@pytest.mark.parametrize("shape", [(2, 36, 516, 40, 9, 1, 4), (2, 36, 516, 40, 9, 2, 4), (2, 36, 517, 40, 7, 1, 3)],
                         ids=["s1", "s2", "s1_ragged_T"])
@pytest.mark.parametrize("algo", CONV1D_ALGOS)
def test_conv1d_inputs_in_guard_regions(algo, shape):
    """The same for op B, at stride 1 and 2 and with T % 4 != 0 (register halo)."""
    case = wl.Conv1dCase("inguard", *shape, seed=8)
    x, dw, pw, bias = wl.conv1d_inputs(case)
    originals = cuda(x, dw, pw, bias)
    guarded = [_guarded_copy(t) for t in originals]
    xg, dwg, pwg, bg = [v for _, v in guarded]
    out = conv1d_or_skip(xg, dwg, pwg, bg, case.stride, case.pad, algo)
    torch.cuda.synchronize()
    _check_guards_and_inputs(guarded, originals)
    ref = oracle.dwsep_conv1d(x.numpy(), dw.numpy(), pw.numpy(), bias.numpy(), case.stride, case.pad)
    assert_close(out, ref, "out")


def test_conv1d_bitwise_repeatable():
    case = wl.CONV1D_SMALL
    x, dw, pw, bias = cuda(*wl.conv1d_inputs(case))
    for algo in CONV1D_ALGOS:
        try:
            a = fcv.dwsep_conv1d(x, dw, pw, bias, case.stride, case.pad, algo=algo)
        except fcv.FcvError as e:
            if e.status == 2:
                continue
            raise
        b_ = fcv.dwsep_conv1d(x, dw, pw, bias, case.stride, case.pad, algo=algo)
        torch.cuda.synchronize()
        assert torch.equal(a, b_)


def test_conv2d_repeatable_within_rounding():
    case = wl.Conv2dCase("rep", 4, 8, 128, 128, 64, 4, seed=13)
    x, w, b = cuda(*wl.conv2d_inputs(case))
    a = fcv.conv2d_pool_sigmoid_sum(x, w, b, case.P)
    b_ = fcv.conv2d_pool_sigmoid_sum(x, w, b, case.P)
    torch.cuda.synchronize()
    assert torch.allclose(a, b_, rtol=1e-6, atol=0)


def test_non_default_stream_and_device_error():
    case = wl.CONV2D_SMALL
    x, w, b = cuda(*wl.conv2d_inputs(case))
    ref = fcv.conv2d_pool_sigmoid_sum(x, w, b, case.P)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out = fcv.conv2d_pool_sigmoid_sum(x, w, b, case.P, stream=s)
    s.synchronize()
    assert torch.allclose(out, ref, rtol=1e-6, atol=0)
    assert fcv.device_error() == 0


def test_host_tensors_through_public_api():
    """CPU inputs: the binding copies to the device, runs the kernel, copies back."""
    case = wl.CONV1D_SMALL
    x, dw, pw, bias = wl.conv1d_inputs(case)
    out = fcv.dwsep_conv1d(x.pin_memory(), dw, pw, bias, case.stride, case.pad)
    assert not out.is_cuda
    assert_close(out, oracle.dwsep_conv1d(x.numpy(), dw.numpy(), pw.numpy(), bias.numpy(), 1, 4), "host conv1d")
    c2 = wl.CONV2D_SMALL
    x2, w2, b2 = wl.conv2d_inputs(c2)
    out2 = fcv.conv2d_pool_sigmoid_sum(x2, w2, b2, c2.P)
    assert not out2.is_cuda
    assert_close(out2, oracle.conv2d_pool_sigmoid_sum(x2.numpy(), w2.numpy(), b2.numpy(), c2.P), "host conv2d")
    # a caller-provided pinned output is filled in place
    dst = torch.full(tuple(out.shape), float("nan"), pin_memory=True)
    got = fcv.dwsep_conv1d(x.pin_memory(), dw, pw, bias, case.stride, case.pad, out=dst)
    assert got.data_ptr() == dst.data_ptr() and torch.equal(dst, out)
    with pytest.raises(ValueError):
        fcv.dwsep_conv1d(x, dw, pw, bias, case.stride, case.pad, out=torch.empty((1,)))


def test_host_tensors_on_a_side_stream():
    """CPU inputs with stream=s and no stream context: the input copies, the
    buffers the binding allocates and the kernel are all ordered on s."""
    s = torch.cuda.Stream()
    c2 = wl.CONV2D_SMALL
    x2, w2, b2 = wl.conv2d_inputs(c2)
    ref2 = oracle.conv2d_pool_sigmoid_sum(x2.numpy(), w2.numpy(), b2.numpy(), c2.P)
    for _ in range(3):
        out2 = fcv.conv2d_pool_sigmoid_sum(x2.pin_memory(), w2, b2, c2.P, stream=s)
        assert_close(out2, ref2, "side-stream conv2d")
    case = wl.CONV1D_SMALL
    x, dw, pw, bias = wl.conv1d_inputs(case)
    out = fcv.dwsep_conv1d(x.pin_memory(), dw, pw, bias, case.stride, case.pad, stream=s)
    assert_close(out, oracle.dwsep_conv1d(x.numpy(), dw.numpy(), pw.numpy(), bias.numpy(), 1, 4), "side-stream conv1d")


def test_empty_batch_through_binding():
    x = torch.zeros((0, 3, 10, 10), device="cuda")
    w = torch.zeros((4, 3, 3, 3), device="cuda")
    b = torch.zeros((4,), device="cuda")
    assert fcv.conv2d_pool_sigmoid_sum(x, w, b, 2).shape == (0,)
    x1 = torch.zeros((0, 3, 10), device="cuda")
    out = fcv.dwsep_conv1d(x1, torch.zeros((3, 3), device="cuda"), torch.zeros((5, 3), device="cuda"), None, 1, 1)
    assert out.shape == (0, 5, 10)


# ------------------------------------------------- op A, deterministic sum ---

@pytest.mark.parametrize("case", [wl.CONV2D_SMALL, wl.CONV2D_FULL,
                                  wl.Conv2dCase("det_odd", 3, 5, 61, 47, 70, 3, seed=17),
                                  wl.Conv2dCase("det_p2", 4, 16, 130, 130, 128, 2, seed=18)],
                         ids=lambda c: c.name)
def test_conv2d_det_parity_and_bitwise_repeatable(case):
    x, w, b = wl.conv2d_inputs(case)
    xd, wd, bd = cuda(x, w, b)
    need = fcv.conv2d_workspace_bytes(case.N, case.Cin, case.H, case.W, case.Cout, case.P)
    ws = torch.full(((need + 15) // 16 * 4,), float("nan"), device="cuda")  # contents on entry do not matter
    first = fcv.conv2d_pool_sigmoid_sum_det(xd, wd, bd, case.P, workspace=ws).clone()
    ws.fill_(123.0)
    second = fcv.conv2d_pool_sigmoid_sum_det(xd, wd, bd, case.P, workspace=ws)
    # the same FMA kernel with atomic adds: equal up to the order of the block sums
    atomic = fcv.conv2d_pool_sigmoid_sum(xd, wd, bd, case.P, algo=fcv.CONV2D_DIRECT)
    auto = fcv.conv2d_pool_sigmoid_sum(xd, wd, bd, case.P)
    torch.cuda.synchronize()
    assert torch.equal(first, second), "deterministic mode differs between runs"
    assert torch.allclose(first, atomic, rtol=1e-6, atol=0)
    assert torch.allclose(first, auto, rtol=1e-5, atol=0)  # AUTO may be the 3xTF32 tensor-core kernel
    xn, wn, bn = x.numpy(), w.numpy(), b.numpy()
    for bi in sorted({0, case.N - 1}):
        assert_close(first[bi:bi + 1], oracle.conv2d_pool_sigmoid_sum(xn[bi:bi + 1], wn, bn, case.P),
                     f"{case.name} det out[{bi}]")


def test_conv2d_det_empty_pool_and_guard_bands():
    case = wl.Conv2dCase("det_empty", 3, 2, 5, 40, 4, 4, seed=9)  # PH = 0: no workspace needed
    x, w, b = cuda(*wl.conv2d_inputs(case))
    assert fcv.conv2d_workspace_bytes(3, 2, 5, 40, 4, 4) == 0
    out = torch.full((3,), 7.0, device="cuda")
    fcv.conv2d_pool_sigmoid_sum_det(x, w, b, 4, out=out)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    guard = 256
    c2 = wl.Conv2dCase("det_guard", 5, 3, 50, 45, 20, 4, seed=10)
    x, w, b = cuda(*wl.conv2d_inputs(c2))
    need = fcv.conv2d_workspace_bytes(c2.N, c2.Cin, c2.H, c2.W, c2.Cout, c2.P)
    wbuf = torch.full((need // 4 + 2 * guard,), float("nan"), device="cuda")
    obuf = torch.full((c2.N + 2 * guard,), float("nan"), device="cuda")
    fcv.conv2d_pool_sigmoid_sum_det(x, w, b, c2.P, out=obuf[guard:guard + c2.N], workspace=wbuf[guard:guard + need // 4])
    torch.cuda.synchronize()
    for buf in (wbuf, obuf):
        assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[-guard:]).all()
    assert torch.isfinite(obuf[guard:guard + c2.N]).all()


# ---------------------------------------------------------- failure path ---

def test_bounded_wait_times_out_and_context_survives():
    """A wait on a barrier nothing completes (2 ms limit) records FCV_ERR_TIMEOUT
    in the device error word; the error is read once and cleared, and the
    context keeps working."""
    lib = fcv.load()
    import ctypes
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.fcv_device_error(stream) == 0
    assert lib.fcv_selftest_wait_timeout(2_000_000, stream) == 0
    assert lib.fcv_device_error(stream) == 4   # FCV_ERR_TIMEOUT
    assert lib.fcv_device_error(stream) == 0   # cleared by the read
    case = wl.CONV1D_SMALL
    check_conv1d_case(case, fcv.CONV1D_TC_3XTF32, n_samples=0)
    assert lib.fcv_device_error(stream) == 0
