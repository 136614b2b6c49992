"""Planted mistakes in the oracle must be caught by its pins.

Each case copies ``oracle/fcv_oracle.c`` to a temporary directory, makes one
plausible mistake there (a dropped term, a wrong sign or index, a transposed
operand, a flipped kernel, ceil instead of floor), compiles the copy and runs
every pin against it.  At least one pin must fail.  The committed oracle is
never modified; a mistake whose target text is missing fails the test, so this
list stays in step with the source.
"""
import os
import shutil

import pytest

import oracle
from oracle.build import SRC, build
from tests import oracle_pins

MUTANTS = [
    # op A: conv stage
    ("conv2d_w_ky_kx_swapped", "const double wv = (double)w[(((size_t)c * Cin + ic) * 3 + ky) * 3 + kx];",
     "const double wv = (double)w[(((size_t)c * Cin + ic) * 3 + kx) * 3 + ky];"),
    ("conv2d_kernel_flipped", "const double wv = (double)w[(((size_t)c * Cin + ic) * 3 + ky) * 3 + kx];",
     "const double wv = (double)w[(((size_t)c * Cin + ic) * 3 + (2 - ky)) * 3 + (2 - kx)];"),
    ("conv2d_input_rows_cols_swapped", "const float* row = xin + (size_t)(y + ky) * W + kx;",
     "const float* row = xin + (size_t)(y + kx) * W + ky;"),
    ("conv2d_bias_dropped", "plane[(size_t)y * Wo + xo] = (double)bias[c];",
     "plane[(size_t)y * Wo + xo] = 0.0;"),
    ("conv2d_wrong_input_channel", "const float* xin = x + ((size_t)b * Cin + ic) * (size_t)H * W;",
     "const float* xin = x + ((size_t)b * Cin + (Cin - 1 - ic)) * (size_t)H * W;"),
    ("conv2d_ky_range_short", "for (int ky = 0; ky < 3; ++ky) {\n            for (int kx = 0; kx < 3; ++kx) {\n                const double wv",
     "for (int ky = 0; ky < 2; ++ky) {\n            for (int kx = 0; kx < 3; ++kx) {\n                const double wv"),
    # op A: pool stage
    ("pool_divisor_P", "return s / ((double)P * (double)P);", "return s / ((double)P);"),
    ("pool_window_not_strided", "s += plane[(size_t)(P * ph + dy) * Wo + (P * pw + dx)];",
     "s += plane[(size_t)(ph + dy) * Wo + (pw + dx)];"),
    ("pool_ceil_mode", "*PH = *Ho / P;", "*PH = (*Ho + P - 1) / P;"),
    # op A: sigmoid and sum
    ("sigmoid_sign", "return 1.0 / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(v));"),
    ("sum_drops_last_channel", "for (int c = 0; c < Cout; ++c) s += partial[(size_t)b * Cout + c];",
     "for (int c = 0; c + 1 < Cout; ++c) s += partial[(size_t)b * Cout + c];"),
    # op A: one-at-a-time path
    ("tap_at_kernel_flipped", "* (double)w[(((size_t)c * Cin + ic) * 3 + ky) * 3 + kx];",
     "* (double)w[(((size_t)c * Cin + ic) * 3 + (2 - ky)) * 3 + kx];"),
    ("tap_at_bias_dropped", "double conv = (double)bias[c];", "double conv = 0.0;"),
    # op B
    ("conv1d_pad_sign", "acc += xpad(xrow, T, (long long)t * s + k - p) * (double)dw[(size_t)c * K + k];",
     "acc += xpad(xrow, T, (long long)t * s + k + p) * (double)dw[(size_t)c * K + k];"),
    ("conv1d_kernel_flipped", "acc += xpad(xrow, T, (long long)t * s + k - p) * (double)dw[(size_t)c * K + k];",
     "acc += xpad(xrow, T, (long long)t * s + k - p) * (double)dw[(size_t)c * K + (K - 1 - k)];"),
    ("conv1d_stride_ignored", "acc += xpad(xrow, T, (long long)t * s + k - p) * (double)dw[(size_t)c * K + k];",
     "acc += xpad(xrow, T, (long long)t + k - p) * (double)dw[(size_t)c * K + k];"),
    ("conv1d_pw_transposed", "const double pv = (double)pw[(size_t)o * C + c];",
     "const double pv = (double)pw[((size_t)o * C + c) % ((size_t)O * C) == 0 ? 0 : ((size_t)c * O + o) % ((size_t)O * C)];"),
    ("conv1d_bias_dropped", "for (int t = 0; t < To; ++t) orow[t] += bo;", "(void)bo;"),
    ("conv1d_replicate_pad", "return (i >= 0 && i < T) ? (double)xrow[i] : 0.0;",
     "return (i >= 0 && i < T) ? (double)xrow[i] : (double)xrow[i < 0 ? 0 : T - 1];"),
    ("conv1d_out_len_no_floor", "*To = (int)(span / s) + 1;", "*To = (int)((span + s - 1) / s) + 1;"),
    ("conv1d_at_pw_wrong_row", "acc += dwsum * (double)pw[(size_t)o * C + c];",
     "acc += dwsum * (double)pw[(size_t)((o + 1) % O) * C + c];"),
    ("conv1d_at_bias_dropped", "vals[i] = acc + (bias ? (double)bias[o] : 0.0);", "vals[i] = acc;"),
]


@pytest.fixture(scope="module")
def src_text():
    with open(SRC) as f:
        return f.read()


def test_committed_oracle_passes_every_pin():
    results = oracle_pins.run_pins(oracle.load())
    assert all(ok for _, ok, _ in results), [r for r in results if not r[1]]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, src_text, name, old, new):
    assert src_text.count(old) == 1, f"mutation target for {name} not found exactly once"
    src = tmp_path / "fcv_oracle_mutant.c"
    src.write_text(src_text.replace(old, new))
    lib_path = str(tmp_path / f"libmutant_{name}.so")
    build(force=True, src=str(src), out=lib_path, werror=False)
    lib = oracle.load(lib_path)
    results = oracle_pins.run_pins(lib)
    failed = [r[0] for r in results if not r[1]]
    assert failed, f"mutant {name} passed every pin"
    shutil.rmtree(tmp_path, ignore_errors=True)
    os.makedirs(tmp_path, exist_ok=True)
