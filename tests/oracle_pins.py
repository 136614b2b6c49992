"""Checks that pin the CPU oracle to facts other than its own code.

Each pin runs the oracle (through a given ctypes handle, so that the mutation
test can point it at a deliberately broken copy) and compares it with one of:

* the shapes the pages print (``tests/golden/shapes.txt``);
* a library routine: torch CPU float64 conv2d / avg_pool2d / sigmoid / sum and
  conv1d(groups=C) / conv1d(1x1);
* brute force on tiny inputs (numpy sliding windows + einsum, a computation
  built differently from the oracle's loops);
* closed forms: impulse responses, zero weights, constant input, zero input,
  the K=1 reduction to a matrix product;
* invariants: linearity, bias folding, the dense fused-weight identity.

A pin returns ``(name, ok, detail)``; none raises on a mismatch.
"""
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "shapes.txt")

# Oracle and library routine both work in double; they differ only in rounding order.
TOL = 1e-10


def _close(a, b, tol=TOL):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.shape != b.shape:
        return False, f"shape {a.shape} vs {b.shape}"
    if a.size == 0:
        return True, "empty"
    err = np.max(np.abs(a - b) / (1.0 + np.abs(b)))
    return bool(err <= tol), f"max scaled err {err:.3e}"


def _rng(seed):
    return np.random.default_rng(seed)


def _grid(a):
    """Round to multiples of 2^-12 so small linear combinations stay exact in fp32."""
    return (np.round(a.astype(np.float64) * 4096.0) / 4096.0).astype(np.float32)


def _conv2d_rand(seed, N, Cin, H, W, Cout):
    r = _rng(seed)
    x = r.standard_normal((N, Cin, H, W)).astype(np.float32)
    bound = 1.0 / math.sqrt(Cin * 9)
    w = r.uniform(-bound, bound, (Cout, Cin, 3, 3)).astype(np.float32)
    b = r.uniform(-bound, bound, (Cout,)).astype(np.float32)
    return x, w, b


def _conv1d_rand(seed, N, C, T, O, K):
    r = _rng(seed)
    x = r.standard_normal((N, C, T)).astype(np.float32)
    dw = r.uniform(-1 / math.sqrt(K), 1 / math.sqrt(K), (C, K)).astype(np.float32)
    pw = r.uniform(-1 / math.sqrt(C), 1 / math.sqrt(C), (O, C)).astype(np.float32)
    bias = r.uniform(-1 / math.sqrt(C), 1 / math.sqrt(C), (O,)).astype(np.float32)
    return x, dw, pw, bias


# ----------------------------------------------------------------------------
# golden shapes printed on the pages
# ----------------------------------------------------------------------------

def read_golden_shapes(path=GOLDEN):
    """Parse ``shapes.txt``: ``conv2d H W P Ho Wo PH PW`` / ``conv1d T K s p To`` rows."""
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            rows.append((parts[0], [int(v) for v in parts[1:]]))
    return rows


def pin_golden_shapes(lib):
    bad = []
    for kind, vals in read_golden_shapes():
        if kind == "conv2d":
            H, W, P, Ho, Wo, PH, PW = vals
            got = oracle.conv2d_out_dims(H, W, P, lib)
            if got != (Ho, Wo, PH, PW):
                bad.append((kind, vals, got))
        elif kind == "conv1d":
            T, K, s, p, To = vals
            got = oracle.conv1d_out_len(T, K, s, p, lib)
            if got != To:
                bad.append((kind, vals, got))
    return "golden_shapes", not bad, str(bad[:3])


# ----------------------------------------------------------------------------
# op A pins
# ----------------------------------------------------------------------------

def _torch_tap(x, w, b, P):
    y = F.conv2d(torch.from_numpy(x).double(), torch.from_numpy(w).double(),
                 torch.from_numpy(b).double())
    return F.avg_pool2d(y, P)  # stride P, padding 0, floor


def pin_conv2d_torch(lib):
    """Tap and scalar against torch float64 on shapes with ragged floors."""
    shapes = [(2, 3, 11, 13, 5, 4), (1, 8, 16, 16, 4, 4), (2, 2, 9, 7, 3, 2),
              (1, 4, 8, 10, 2, 3), (1, 1, 5, 5, 1, 1), (3, 5, 14, 12, 6, 5)]
    for i, (N, Cin, H, W, Cout, P) in enumerate(shapes):
        x, w, b = _conv2d_rand(100 + i, N, Cin, H, W, Cout)
        ref = _torch_tap(x, w, b, P)
        ok, d = _close(oracle.conv2d_pool_tap(x, w, b, P, lib), ref.numpy())
        if not ok:
            return "conv2d_torch_tap", False, f"{(N, Cin, H, W, Cout, P)}: {d}"
        ok, d = _close(oracle.conv2d_pool_sigmoid_sum(x, w, b, P, lib),
                       torch.sigmoid(ref).sum(dim=(1, 2, 3)).numpy())
        if not ok:
            return "conv2d_torch_sum", False, f"{(N, Cin, H, W, Cout, P)}: {d}"
    return "conv2d_torch", True, ""


def pin_conv2d_bruteforce(lib):
    """Tiny shapes against numpy sliding windows + einsum + block mean."""
    from numpy.lib.stride_tricks import sliding_window_view
    for i, (N, Cin, H, W, Cout, P) in enumerate([(2, 3, 10, 9, 4, 2), (1, 2, 7, 11, 3, 3)]):
        x, w, b = _conv2d_rand(200 + i, N, Cin, H, W, Cout)
        win = sliding_window_view(x.astype(np.float64), (3, 3), axis=(2, 3))
        conv = np.einsum("nchwij,ocij->nohw", win, w.astype(np.float64)) + b.astype(np.float64)[None, :, None, None]
        PH, PW = conv.shape[2] // P, conv.shape[3] // P
        pooled = conv[:, :, :PH * P, :PW * P].reshape(N, Cout, PH, P, PW, P).mean(axis=(3, 5))
        ok, d = _close(oracle.conv2d_pool_tap(x, w, b, P, lib), pooled)
        if not ok:
            return "conv2d_bruteforce_tap", False, d
        total = (1.0 / (1.0 + np.exp(-pooled))).sum(axis=(1, 2, 3))
        ok, d = _close(oracle.conv2d_pool_sigmoid_sum(x, w, b, P, lib), total)
        if not ok:
            return "conv2d_bruteforce_sum", False, d
    return "conv2d_bruteforce", True, ""


def pin_conv2d_impulse(lib):
    """x = delta at (ic0, y0, x0), bias 0, P = 1: tap[c, y, x] = w[c, ic0, y0-y, x0-x]."""
    N, Cin, H, W, Cout = 1, 3, 8, 9, 4
    _, w, _ = _conv2d_rand(300, N, Cin, H, W, Cout)
    b = np.zeros((Cout,), np.float32)
    for (ic0, y0, x0) in [(0, 0, 0), (1, 4, 5), (2, 7, 8), (1, 2, 1)]:
        x = np.zeros((N, Cin, H, W), np.float32)
        x[0, ic0, y0, x0] = 1.0
        want = np.zeros((N, Cout, H - 2, W - 2))
        for y in range(H - 2):
            for xx in range(W - 2):
                ky, kx = y0 - y, x0 - xx
                if 0 <= ky < 3 and 0 <= kx < 3:
                    want[0, :, y, xx] = w[:, ic0, ky, kx]
        ok, d = _close(oracle.conv2d_pool_tap(x, w, b, 1, lib), want)
        if not ok:
            return "conv2d_impulse", False, f"delta {(ic0, y0, x0)}: {d}"
    # the same delta through P = 2 averages the 2x2 windows of that response
    x = np.zeros((N, Cin, H, W), np.float32)
    x[0, 1, 4, 5] = 1.0
    resp = oracle.conv2d_pool_tap(x, w, b, 1, lib)
    want = resp[:, :, :6, :6].reshape(N, Cout, 3, 2, 3, 2).mean(axis=(3, 5))
    ok, d = _close(oracle.conv2d_pool_tap(x, w, b, 2, lib), want)
    return "conv2d_impulse", ok, d


def pin_conv2d_zero_weights(lib):
    """w = 0: out[b] = PH * PW * sum_c sigmoid(bias[c]); equal biases give Cout*PH*PW*sigmoid(b)."""
    N, Cin, H, W, Cout, P = 2, 3, 13, 10, 5, 3
    x, w, b = _conv2d_rand(400, N, Cin, H, W, Cout)
    w[:] = 0.0
    PH, PW = (H - 2) // P, (W - 2) // P
    want = PH * PW * np.sum(1.0 / (1.0 + np.exp(-b.astype(np.float64))))
    ok, d = _close(oracle.conv2d_pool_sigmoid_sum(x, w, b, P, lib), np.full((N,), want), 1e-12)
    if not ok:
        return "conv2d_zero_weights", False, d
    b[:] = np.float32(0.25)
    want = Cout * PH * PW / (1.0 + math.exp(-float(np.float32(0.25))))
    ok, d = _close(oracle.conv2d_pool_sigmoid_sum(x, w, b, P, lib), np.full((N,), want), 1e-12)
    return "conv2d_zero_weights", ok, d


def pin_conv2d_constant_input(lib):
    """x = kappa everywhere: every pooled value is bias[c] + kappa * sum(w[c])."""
    N, Cin, H, W, Cout, P = 1, 4, 11, 9, 3, 2
    _, w, b = _conv2d_rand(500, N, Cin, H, W, Cout)
    kappa = 0.75
    x = np.full((N, Cin, H, W), kappa, np.float32)
    per_c = b.astype(np.float64) + kappa * w.astype(np.float64).reshape(Cout, -1).sum(axis=1)
    PH, PW = (H - 2) // P, (W - 2) // P
    want = np.broadcast_to(per_c[None, :, None, None], (N, Cout, PH, PW))
    ok, d = _close(oracle.conv2d_pool_tap(x, w, b, P, lib), want)
    return "conv2d_constant_input", ok, d


def pin_conv2d_ramp_floor(lib):
    """x[y, x] = y (a ramp) with floored pooling.

    conv[y] = bias + sum_{ic,ky,kx} w * (y + ky), linear in y; the pooled row ph
    averages conv rows P*ph .. P*ph+P-1, so it equals conv at y = P*ph + (P-1)/2.
    Rows past PH*P are dropped: with H = 11, P = 4 the 9 conv rows give 2 pooled
    rows.  Checks window placement, the divisor and the floor.
    """
    N, Cin, H, W, Cout, P = 1, 2, 11, 11, 3, 4
    _, w, b = _conv2d_rand(600, N, Cin, H, W, Cout)
    x = np.broadcast_to(np.arange(H, dtype=np.float32)[None, None, :, None], (N, Cin, H, W)).copy()
    w64 = w.astype(np.float64)
    s0 = w64.reshape(Cout, -1).sum(axis=1)
    s1 = np.einsum("ocij,i->o", w64, np.arange(3, dtype=np.float64))
    PH = (H - 2) // P
    want = np.zeros((N, Cout, PH, PH))
    for ph in range(PH):
        yc = P * ph + (P - 1) / 2.0
        want[0, :, ph, :] = (b.astype(np.float64) + s0 * yc + s1)[:, None]
    ok, d = _close(oracle.conv2d_pool_tap(x, w, b, P, lib), want)
    return "conv2d_ramp_floor", ok, d


def pin_conv2d_linearity_and_bias(lib):
    """tap(a*x1 + c*x2) - bias = a(tap(x1) - bias) + c(tap(x2) - bias); tap(w, b) = tap(w, 0) + b."""
    N, Cin, H, W, Cout, P = 2, 3, 12, 14, 4, 3
    x1, w, b = _conv2d_rand(700, N, Cin, H, W, Cout)
    x2, _, _ = _conv2d_rand(701, N, Cin, H, W, Cout)
    x1, x2 = _grid(x1), _grid(x2)
    a, c = 0.5, -2.0  # with inputs on a 2^-12 grid, a*x1 + c*x2 is exact in fp32
    x3 = (a * x1.astype(np.float64) + c * x2.astype(np.float64)).astype(np.float32)
    bb = b.astype(np.float64)[None, :, None, None]
    t1 = oracle.conv2d_pool_tap(x1, w, b, P, lib) - bb
    t2 = oracle.conv2d_pool_tap(x2, w, b, P, lib) - bb
    t3 = oracle.conv2d_pool_tap(x3, w, b, P, lib) - bb
    ok, d = _close(t3, a * t1 + c * t2, 1e-9)
    if not ok:
        return "conv2d_linearity", False, d
    t0 = oracle.conv2d_pool_tap(x1, w, np.zeros_like(b), P, lib)
    ok, d = _close(t1, t0)
    return "conv2d_bias_folding", ok, d


def pin_conv2d_empty_pool(lib):
    """Fewer conv rows than P: PH = 0, so the sum is over an empty set and out = 0."""
    x, w, b = _conv2d_rand(800, 2, 2, 5, 9, 3)
    out = oracle.conv2d_pool_sigmoid_sum(x, w, b, 4, lib)  # Ho = 3 < 4
    tap = oracle.conv2d_pool_tap(x, w, b, 4, lib)
    ok = bool(np.all(out == 0.0)) and tap.shape == (2, 3, 0, 1)
    return "conv2d_empty_pool", ok, f"{out} {tap.shape}"


def pin_conv2d_tap_at(lib):
    """The one-at-a-time path against torch float64 at sampled indices."""
    N, Cin, H, W, Cout, P = 2, 5, 23, 19, 6, 4
    x, w, b = _conv2d_rand(900, N, Cin, H, W, Cout)
    ref = _torch_tap(x, w, b, P).numpy()
    r = _rng(901)
    idx = np.stack([r.integers(0, s, 64) for s in ref.shape], axis=1)
    want = ref[idx[:, 0], idx[:, 1], idx[:, 2], idx[:, 3]]
    ok, d = _close(oracle.conv2d_pool_tap_at(x, w, b, P, idx, lib), want)
    return "conv2d_tap_at", ok, d


# ----------------------------------------------------------------------------
# op B pins
# ----------------------------------------------------------------------------

def _torch_dwsep(x, dw, pw, bias, s, p):
    C, K = dw.shape
    O = pw.shape[0]
    d = F.conv1d(torch.from_numpy(x).double(), torch.from_numpy(dw).double().view(C, 1, K),
                 stride=s, padding=p, groups=C)
    bt = None if bias is None else torch.from_numpy(bias).double()
    return F.conv1d(d, torch.from_numpy(pw).double().view(O, C, 1), bt)


def pin_conv1d_torch(lib):
    """Two-stage oracle against torch float64 conv1d(groups=C) then 1x1 conv."""
    for i, (N, C, T, O, K, s, p, nb) in enumerate([
            (2, 4, 17, 5, 3, 1, 1, False), (1, 6, 33, 3, 9, 1, 4, False), (2, 3, 20, 4, 5, 2, 2, False),
            (1, 5, 9, 2, 9, 2, 0, False), (1, 3, 40, 7, 4, 3, 3, True), (2, 2, 5, 3, 7, 1, 5, False)]):
        x, dw, pw, bias = _conv1d_rand(1000 + i, N, C, T, O, K)
        if nb:
            bias = None
        ok, d = _close(oracle.dwsep_conv1d(x, dw, pw, bias, s, p, lib), _torch_dwsep(x, dw, pw, bias, s, p).numpy())
        if not ok:
            return "conv1d_torch", False, f"{(N, C, T, O, K, s, p)}: {d}"
    return "conv1d_torch", True, ""


def pin_conv1d_dense_fused_weight(lib):
    """W[o,c,k] = dw[c,k] * pw[o,c] turns the op into one dense conv1d (torch float64)."""
    N, C, T, O, K, s, p = 2, 5, 31, 6, 9, 2, 4
    x, dw, pw, bias = _conv1d_rand(1100, N, C, T, O, K)
    Wd = torch.from_numpy(pw).double()[:, :, None] * torch.from_numpy(dw).double()[None, :, :]
    ref = F.conv1d(torch.from_numpy(x).double(), Wd, torch.from_numpy(bias).double(), stride=s, padding=p)
    ok, d = _close(oracle.dwsep_conv1d(x, dw, pw, bias, s, p, lib), ref.numpy())
    if not ok:
        return "conv1d_dense_fused_weight", False, d
    r = _rng(1101)
    idx = np.stack([r.integers(0, n, 48) for n in ref.shape], axis=1)
    want = ref.numpy()[idx[:, 0], idx[:, 1], idx[:, 2]]
    ok, d = _close(oracle.dwsep_conv1d_at(x, dw, pw, bias, s, p, idx, lib), want)
    return "conv1d_dense_fused_weight_at", ok, d


def pin_conv1d_impulse(lib):
    """x = delta(b0,c0,t0), bias 0: out[b0,o,t] = pw[o,c0]*dw[c0, t0 - t*s + p] when in range."""
    N, C, T, O, K = 2, 3, 19, 4, 5
    _, dw, pw, _ = _conv1d_rand(1200, N, C, T, O, K)
    for (b0, c0, t0, s, p) in [(0, 0, 0, 1, 2), (1, 2, 18, 1, 2), (1, 1, 7, 2, 3), (0, 2, 10, 3, 0)]:
        x = np.zeros((N, C, T), np.float32)
        x[b0, c0, t0] = 1.0
        To = (T + 2 * p - K) // s + 1
        want = np.zeros((N, O, To))
        for t in range(To):
            k = t0 - t * s + p
            if 0 <= k < K:
                want[b0, :, t] = pw[:, c0].astype(np.float64) * float(dw[c0, k])
        ok, d = _close(oracle.dwsep_conv1d(x, dw, pw, None, s, p, lib), want)
        if not ok:
            return "conv1d_impulse", False, f"{(b0, c0, t0, s, p)}: {d}"
        idx = np.array([[b0, o, t] for o in range(O) for t in range(To)])
        ok, d = _close(oracle.dwsep_conv1d_at(x, dw, pw, None, s, p, idx, lib), want[b0].reshape(-1))
        if not ok:
            return "conv1d_impulse_at", False, f"{(b0, c0, t0, s, p)}: {d}"
    return "conv1d_impulse", True, ""


def pin_conv1d_linearity_zero(lib):
    """Linear in x when bias is absent; x = 0 gives the bias broadcast along t."""
    N, C, T, O, K, s, p = 2, 4, 25, 3, 9, 1, 4
    x1, dw, pw, bias = _conv1d_rand(1300, N, C, T, O, K)
    x2, _, _, _ = _conv1d_rand(1301, N, C, T, O, K)
    x1, x2 = _grid(x1), _grid(x2)
    a, c = 2.0, -0.25  # exact: inputs on a 2^-12 grid
    x3 = (a * x1.astype(np.float64) + c * x2.astype(np.float64)).astype(np.float32)
    f = lambda z: oracle.dwsep_conv1d(z, dw, pw, None, s, p, lib)
    ok, d = _close(f(x3), a * f(x1) + c * f(x2), 1e-9)
    if not ok:
        return "conv1d_linearity", False, d
    z = oracle.dwsep_conv1d(np.zeros_like(x1), dw, pw, bias, s, p, lib)
    ok, d = _close(z, np.broadcast_to(bias.astype(np.float64)[None, :, None], z.shape), 0.0)
    return "conv1d_zero_input", ok, d


def pin_conv1d_k1_gemm(lib):
    """K = 1, p = 0, s = 1: out[b] = pw @ diag(dw) @ x[b] + bias (numpy matmul)."""
    N, C, T, O = 3, 6, 11, 5
    x, dw, pw, bias = _conv1d_rand(1400, N, C, T, O, 1)
    want = np.einsum("oc,btc->bot", pw.astype(np.float64) * dw[:, 0].astype(np.float64)[None, :],
                     np.transpose(x, (0, 2, 1)).astype(np.float64)) + bias.astype(np.float64)[None, :, None]
    ok, d = _close(oracle.dwsep_conv1d(x, dw, pw, bias, 1, 0, lib), want)
    return "conv1d_k1_gemm", ok, d


def pin_conv1d_at_matches_full(lib):
    """Fused order (one output at a time) against the two-stage oracle, stride 2, ragged T."""
    N, C, T, O, K, s, p = 2, 7, 37, 5, 9, 2, 4
    x, dw, pw, bias = _conv1d_rand(1500, N, C, T, O, K)
    full = oracle.dwsep_conv1d(x, dw, pw, bias, s, p, lib)
    r = _rng(1501)
    idx = np.stack([r.integers(0, n, 64) for n in full.shape], axis=1)
    idx[0] = [0, 0, 0]
    idx[1] = [N - 1, O - 1, full.shape[2] - 1]
    ok, d = _close(oracle.dwsep_conv1d_at(x, dw, pw, bias, s, p, idx, lib),
                   full[idx[:, 0], idx[:, 1], idx[:, 2]])
    return "conv1d_at_matches_full", ok, d


CONV2D_PINS = [pin_conv2d_torch, pin_conv2d_bruteforce, pin_conv2d_impulse, pin_conv2d_zero_weights,
               pin_conv2d_constant_input, pin_conv2d_ramp_floor, pin_conv2d_linearity_and_bias,
               pin_conv2d_empty_pool, pin_conv2d_tap_at]
CONV1D_PINS = [pin_conv1d_torch, pin_conv1d_dense_fused_weight, pin_conv1d_impulse,
               pin_conv1d_linearity_zero, pin_conv1d_k1_gemm, pin_conv1d_at_matches_full]
ALL_PINS = [pin_golden_shapes] + CONV2D_PINS + CONV1D_PINS


def run_pins(lib, pins=ALL_PINS):
    """Run pins, turning a crash inside a broken oracle into a failed pin."""
    results = []
    for pin in pins:
        try:
            results.append(pin(lib))
        except Exception as e:  # a broken oracle may also fail by raising
            results.append((pin.__name__, False, f"raised {type(e).__name__}: {e}"))
    return results
