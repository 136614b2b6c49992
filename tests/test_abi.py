"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments synchronously before touching the
device (these calls return before any CUDA API call)."""
import ctypes
import os
import re
import subprocess

import pytest

from direct_convolution_chip_b200 import binding
from direct_convolution_chip_b200 import build as fcv_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fcv.h")

OK, INVALID, UNSUPPORTED = 0, 1, 2
P = ctypes.c_void_p
FAKE = P(0x10000)     # never dereferenced: every call below returns during validation
MISALIGNED = P(0x10002)
ALIGNED4 = P(0x10004)  # 4-byte aligned, not 16-byte aligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fcv_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    fcv_build.build()
    return binding.load()


def test_header_declares_the_two_ops():
    names = declared_functions()
    assert "fcv_conv2d_pool_sigmoid_sum" in names and "fcv_dwsep_conv1d" in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.lib_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fcv_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    assert set(binding.SIGNATURES) == set(declared_functions())


def test_version_and_status_strings(lib):
    assert lib.fcv_version() >= 100
    for st in range(5):
        assert lib.fcv_status_string(st).decode().startswith(binding.STATUS_NAMES[st])
    assert b"unknown" in lib.fcv_status_string(99)


def c2d(lib, x=FAKE, w=FAKE, b=FAKE, N=2, Cin=8, H=64, W=64, Cout=16, pool=4, out=FAKE, algo=0):
    return lib.fcv_conv2d_pool_sigmoid_sum_ex(x, w, b, N, Cin, H, W, Cout, pool, out, algo, None)


def c1d(lib, x=FAKE, dw=FAKE, pw=FAKE, bias=FAKE, N=2, C=8, T=64, O=16, K=9, s=1, p=4, out=FAKE, algo=0):
    return lib.fcv_dwsep_conv1d_ex(x, dw, pw, bias, N, C, T, O, K, s, p, out, algo, None)


@pytest.mark.parametrize("kw", [
    dict(x=None), dict(w=None), dict(b=None), dict(out=None),
    dict(N=-1), dict(Cin=0), dict(Cout=0), dict(H=2), dict(W=2), dict(pool=0),
    dict(x=MISALIGNED), dict(out=MISALIGNED),
    dict(N=1 << 30, Cin=1 << 30, H=1 << 20, W=1 << 20),  # element count overflows int64
    dict(algo=999), dict(algo=21), dict(algo=14),
])
def test_conv2d_invalid(lib, kw):
    assert c2d(lib, **kw) == INVALID


@pytest.mark.parametrize("kw", [dict(Cin=17), dict(pool=3), dict(x=ALIGNED4)])
def test_conv2d_shifted_tensor_core_envelope(lib, kw):
    """The shifted-operand tensor-core kernel takes Cin <= 16, pool 1/2/4/8 and a
    16-byte aligned x; outside that an explicit request is UNSUPPORTED."""
    assert c2d(lib, algo=13, **kw) == UNSUPPORTED


def stall2d(lib, role=1, at=0, limit=1000, **kw):
    a = dict(x=FAKE, w=FAKE, b=FAKE, N=2, Cin=8, H=64, W=64, Cout=16, pool=4, out=FAKE)
    a.update(kw)
    return lib.fcv_selftest_conv2d_stall(a["x"], a["w"], a["b"], a["N"], a["Cin"], a["H"], a["W"], a["Cout"],
                                         a["pool"], a["out"], role, at, limit, None)


def stall1d(lib, role=1, at=0, limit=1000, **kw):
    a = dict(x=FAKE, dw=FAKE, pw=FAKE, bias=FAKE, N=2, C=32, T=64, O=16, K=9, s=1, p=4, out=FAKE)
    a.update(kw)
    return lib.fcv_selftest_conv1d_stall(a["x"], a["dw"], a["pw"], a["bias"], a["N"], a["C"], a["T"], a["O"], a["K"],
                                         a["s"], a["p"], a["out"], role, at, limit, None)


@pytest.mark.parametrize("fn", [stall2d, stall1d])
@pytest.mark.parametrize("kw,want", [(dict(role=0), "inv"), (dict(role=5), "inv"), (dict(at=-1), "inv"),
                                     (dict(limit=0), "inv"), (dict(limit=11 * 10**9), "inv"), (dict(N=0), "ok")])
def test_stall_selftests_validate_on_the_host(lib, fn, kw, want):
    """The failure-path test entry points reject bad roles, units and limits
    before any CUDA call (N == 0 enqueues nothing)."""
    assert fn(lib, **kw) == {"inv": INVALID, "ok": OK}[want]


def stall1d_pair(lib, role=1, at=0, rank=0, limit=1000, **kw):
    a = dict(x=FAKE, dw=FAKE, pw=FAKE, bias=FAKE, N=2, C=256, T=64, O=256, K=9, s=1, p=4, out=FAKE)
    a.update(kw)
    return lib.fcv_selftest_conv1d_pair_stall(a["x"], a["dw"], a["pw"], a["bias"], a["N"], a["C"], a["T"], a["O"],
                                              a["K"], a["s"], a["p"], a["out"], role, at, rank, limit, None)


@pytest.mark.parametrize("kw,want", [(dict(role=0), "inv"), (dict(role=7), "inv"), (dict(rank=2), "inv"),
                                     (dict(rank=-1), "inv"), (dict(role=3, rank=1), "inv"),
                                     (dict(role=6, rank=0), "inv"), (dict(at=-1), "inv"), (dict(limit=0), "inv"),
                                     (dict(limit=11 * 10**9), "inv"), (dict(N=0), "ok"),
                                     (dict(role=6, rank=1, N=0), "ok"), (dict(role=5, rank=1, N=0), "ok"),
                                     (dict(role=5, s=2), "inv"), (dict(role=6, rank=1, s=2, N=0), "ok")])
def test_pair_stall_selftest_validates_on_the_host(lib, kw, want):
    """The SM-pair failure-path entry point rejects bad roles, ranks (the
    MMA issuer lives in rank 0, the relay in rank 1; the pw split warps work
    at stride 1 only), tiles and limits before any CUDA call."""
    assert stall1d_pair(lib, **kw) == {"inv": INVALID, "ok": OK}[want]


def test_stall_selftests_outside_their_kernels(lib):
    assert stall1d_pair(lib, s=3) == UNSUPPORTED
    assert stall1d_pair(lib, T=66) == UNSUPPORTED
    assert stall2d(lib, Cin=20) == UNSUPPORTED
    assert stall1d(lib, s=3) == UNSUPPORTED


def test_conv2d_unsupported_pool(lib):
    assert c2d(lib, pool=9) == UNSUPPORTED


def test_conv2d_empty_batch_is_a_noop(lib):
    assert c2d(lib, N=0) == OK
    assert c2d(lib, N=0, x=None, w=None, b=None, out=None) == OK  # empty tensors may be NULL
    assert lib.fcv_conv2d_pool_tap(FAKE, FAKE, FAKE, 0, 3, 9, 9, 4, 2, FAKE, 0, None) == OK


def test_conv2d_tap_null_when_pool_is_empty(lib):
    # Ho = 3 < pool 4: the tap has no elements, so it may be NULL; the sum output may not.
    assert lib.fcv_conv2d_pool_tap(FAKE, FAKE, FAKE, 2, 3, 5, 40, 4, 4, None, 0, None) == OK
    assert c2d(lib, H=5, pool=4, out=None) == INVALID


@pytest.mark.parametrize("kw", [
    dict(x=None), dict(dw=None), dict(pw=None), dict(out=None),
    dict(N=-1), dict(C=0), dict(O=0), dict(T=0), dict(K=0), dict(s=0), dict(p=-1),
    dict(T=4, K=9, p=0),  # To < 1
    dict(x=MISALIGNED), dict(bias=MISALIGNED),
    dict(algo=10), dict(algo=7),
])
def test_conv1d_invalid(lib, kw):
    assert c1d(lib, **kw) == INVALID


@pytest.mark.parametrize("kw", [dict(K=33, p=16), dict(s=9), dict(p=1 << 20)])
def test_conv1d_unsupported(lib, kw):
    assert c1d(lib, **kw) == UNSUPPORTED


def test_conv1d_empty_batch_and_null_bias(lib):
    assert c1d(lib, N=0) == OK
    assert c1d(lib, N=0, bias=None) == OK
    assert c1d(lib, N=0, x=None, dw=None, pw=None, out=None) == OK


def test_binding_raises_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        binding.load(str(tmp_path / "missing.so"))


def test_det_workspace_bytes(lib):
    v = ctypes.c_size_t()
    # x[128,8,384,384], Cout 64, pool 4: 12 x 12 tiles of 8x8 pooled outputs, one channel block
    assert lib.fcv_conv2d_workspace_bytes(128, 8, 384, 384, 64, 4, ctypes.byref(v)) == OK
    assert v.value == 128 * 144 * 4 + 128 * 4
    assert lib.fcv_conv2d_workspace_bytes(2, 3, 5, 40, 4, 4, ctypes.byref(v)) == OK and v.value == 0  # PH = 0
    assert lib.fcv_conv2d_workspace_bytes(0, 3, 9, 9, 4, 2, ctypes.byref(v)) == OK and v.value == 0
    assert lib.fcv_conv2d_workspace_bytes(1, 3, 9, 9, 4, 9, ctypes.byref(v)) == UNSUPPORTED
    assert lib.fcv_conv2d_workspace_bytes(1, 0, 9, 9, 4, 2, ctypes.byref(v)) == INVALID
    assert lib.fcv_conv2d_workspace_bytes(1, 3, 9, 9, 4, 2, None) == INVALID


def test_det_rejects_missing_or_small_workspace(lib):
    det = lib.fcv_conv2d_pool_sigmoid_sum_det
    args = (FAKE, FAKE, FAKE, 2, 8, 64, 64, 16, 4, FAKE)
    assert det(*args, None, 1 << 20, None) == INVALID          # workspace needed
    assert det(*args, P(0x10008), 1 << 20, None) == INVALID    # not 16-byte aligned
    assert det(*args, FAKE, 8, None) == INVALID                # too small
    assert det(FAKE, FAKE, FAKE, 0, 8, 64, 64, 16, 4, FAKE, None, 0, None) == OK  # empty batch


def test_selftest_rejects_bad_limits(lib):
    assert lib.fcv_selftest_wait_timeout(0, None) == INVALID
    assert lib.fcv_selftest_wait_timeout(11 * 10**9, None) == INVALID


def test_auto_algo_conv2d(lib):
    """AUTO: FMA for narrow layers (Cin <= 4 and Cout <= 32) once the FMA grid
    has 128 CTAs; else the shifted-operand tensor-core kernel (Cin <= 16, pool
    1, 2, 4 or 8), else the im2col tensor-core kernel where it fits, else FMA."""
    a = ctypes.c_int()
    q = lib.fcv_conv2d_auto_algo
    assert q(128, 8, 384, 384, 64, 4, ctypes.byref(a)) == OK and a.value == 13  # the full-size workload
    for pool in (1, 2, 8):
        assert q(2, 8, 40, 40, 48, pool, ctypes.byref(a)) == OK and a.value == 13
    # narrow layers (Cin <= 4 and Cout <= 32): FMA once its grid has 128 CTAs
    assert q(16, 3, 130, 130, 32, 4, ctypes.byref(a)) == OK and a.value == 10   # exactly 128
    assert q(15, 3, 130, 130, 32, 4, ctypes.byref(a)) == OK and a.value == 13   # 120
    assert q(16, 3, 509, 509, 32, 4, ctypes.byref(a)) == OK and a.value == 10
    assert q(16, 4, 509, 509, 16, 2, ctypes.byref(a)) == OK and a.value == 10
    assert q(16, 3, 509, 509, 48, 4, ctypes.byref(a)) == OK and a.value == 13   # Cout > 32
    assert q(16, 16, 509, 509, 32, 4, ctypes.byref(a)) == OK and a.value == 13  # Cin > 4
    assert q(16, 5, 130, 130, 16, 4, ctypes.byref(a)) == OK and a.value == 13
    assert q(2, 3, 40, 40, 32, 4, ctypes.byref(a)) == OK and a.value == 13      # 8 FMA CTAs: tensor cores
    assert q(2, 8, 64, 64, 16, 4, ctypes.byref(a)) == OK and a.value == 13      # the small workload
    assert q(2, 8, 40, 40, 128, 4, ctypes.byref(a)) == OK and a.value == 13     # two launches of 64 channels
    assert q(2, 20, 40, 40, 48, 4, ctypes.byref(a)) == OK and a.value == 12     # Cin > 16: im2col kernel
    assert q(2, 8, 40, 40, 16, 3, ctypes.byref(a)) == OK and a.value == 10      # pool 3: FMA path
    assert q(2, 40, 40, 40, 128, 4, ctypes.byref(a)) == OK and a.value == 10    # neither tensor-core kernel
    assert q(2, 3, 40, 40, 16, 9, ctypes.byref(a)) == UNSUPPORTED
    assert q(2, 0, 40, 40, 16, 4, ctypes.byref(a)) == INVALID
    assert q(2, 3, 40, 40, 16, 4, None) == INVALID


def test_auto_algo_conv1d(lib):
    """AUTO: the SM-pair kernel for C >= 256 with O >= 256 at stride 1 or any O
    at stride 2 (aligned x/pw, T % 4 == 0), then TMA-halo tensor cores for aligned x/pw, T % 4 == 0
    and stride 1 or 2, then the register-halo tensor-core kernel (stride 1),
    then FMA."""
    a = ctypes.c_int()
    q = lib.fcv_dwsep_conv1d_auto_algo
    X, PW = P(0x10000), P(0x20000)
    assert q(X, PW, 32, 256, 4096, 512, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 22  # full-size workload
    assert q(X, PW, 8, 384, 1000, 768, 3, 1, 1, ctypes.byref(a)) == OK and a.value == 22   # SM pair
    assert q(X, PW, 8, 64, 1000, 768, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 23    # C < 256
    assert q(X, PW, 8, 384, 1000, 128, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 23   # O < 256
    assert q(X, PW, 8, 384, 1000, 768, 9, 2, 4, ctypes.byref(a)) == OK and a.value == 22   # stride 2, SM pair
    assert q(X, PW, 8, 384, 1000, 128, 9, 2, 4, ctypes.byref(a)) == OK and a.value == 22   # stride 2, O = 128
    assert q(X, PW, 8, 64, 1000, 768, 9, 2, 4, ctypes.byref(a)) == OK and a.value == 23    # stride 2, C < 256
    assert q(X, PW, 8, 384, 1001, 768, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 21   # T % 4 != 0
    assert q(P(0x10004), PW, 8, 384, 1000, 768, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 21  # x misaligned
    assert q(X, PW, 2, 64, 1001, 128, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 21    # T % 4 != 0
    assert q(P(0x10004), PW, 2, 64, 1000, 128, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 21  # x not 16-B aligned
    assert q(X, PW, 2, 64, 1000, 128, 9, 2, 4, ctypes.byref(a)) == OK and a.value == 23    # stride 2
    assert q(X, PW, 2, 64, 1001, 128, 9, 2, 4, ctypes.byref(a)) == OK and a.value == 20    # stride 2, T % 4 != 0
    assert q(X, PW, 2, 64, 1000, 128, 9, 3, 4, ctypes.byref(a)) == OK and a.value == 20    # stride 3
    assert q(X, PW, 2, 62, 1000, 128, 9, 1, 4, ctypes.byref(a)) == OK and a.value == 20    # C % 4 != 0
    assert q(X, PW, 2, 64, 1000, 128, 33, 1, 4, ctypes.byref(a)) == UNSUPPORTED           # K > 32
    assert q(X, PW, 2, 64, 1000, 128, 9, 1, -1, ctypes.byref(a)) == INVALID
    assert q(X, PW, 2, 64, 1000, 128, 9, 1, 4, None) == INVALID


def test_binding_calls_run_on_their_stream_argument(monkeypatch):
    """The binding enters torch's stream context for a given `stream` (passed by
    keyword or position), so host copies, allocations and the kernel share it;
    without one it calls straight through."""
    seen = []

    class FakeStreamContext:
        def __init__(self, stream):
            self.stream = stream

        def __enter__(self):
            seen.append(self.stream)

        def __exit__(self, *exc):
            return False

    monkeypatch.setattr(binding.torch.cuda, "stream", FakeStreamContext)

    @binding._on_stream
    def call(a, b=1, stream=None):
        return a, b, stream

    assert call(1) == (1, 1, None) and seen == []
    assert call(1, 2, "s1") == (1, 2, "s1") and seen == ["s1"]
    assert call(1, stream="s2") == (1, 1, "s2") and seen == ["s1", "s2"]
    assert call(1, 3) == (1, 3, None) and seen == ["s1", "s2"]


def test_conv2d_tc_plan_fits_tensor_memory_and_shared_memory(lib):
    """For every shape the tensor-core conv2d accepts, the launch plan stays
    within the 512 TMEM columns the kernel allocates and the 227 KB of shared
    memory a CTA may request; the sub-chunk kernel runs exactly where it
    applies (TMA halo, Cout rounded to 16 at most 96)."""
    v, n, t, sm = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_uint()
    q = lib.fcv_conv2d_tc_plan
    supported = 0
    for cin in (1, 3, 8, 9, 16, 24, 32, 40, 48, 64, 65):
        for cout in range(1, 121):
            for pool in (1, 2, 4, 8):
                for tma in (0, 1):
                    st = q(cin, cout, pool, tma, ctypes.byref(v), ctypes.byref(n), ctypes.byref(t), ctypes.byref(sm))
                    if cout > 112:
                        assert st == UNSUPPORTED
                        continue
                    if st == UNSUPPORTED:
                        continue  # weights too large for shared memory
                    assert st == OK
                    supported += 1
                    np_ = (cout + 15) // 16 * 16
                    assert v.value == int(bool(tma) and np_ <= 96)
                    a_cols = 4 * 80 if v.value else 2 * 144
                    assert n.value in (2, 3) and t.value == n.value * np_ + a_cols <= 512
                    assert n.value == (3 if 3 * np_ + a_cols <= 512 else 2)
                    assert 120 * 1024 <= sm.value <= 227 * 1024
    assert supported > 3000
    # the full-size workload: sub-chunk kernel, three accumulators, all 512 columns
    assert q(8, 64, 4, 1, ctypes.byref(v), ctypes.byref(n), ctypes.byref(t), ctypes.byref(sm)) == OK
    assert (v.value, n.value, t.value) == (1, 3, 512)
    assert q(8, 64, 3, 1, ctypes.byref(v), ctypes.byref(n), ctypes.byref(t), ctypes.byref(sm)) == UNSUPPORTED
    assert q(0, 64, 4, 1, ctypes.byref(v), ctypes.byref(n), ctypes.byref(t), ctypes.byref(sm)) == INVALID
    assert q(8, 64, 4, 1, None, ctypes.byref(n), ctypes.byref(t), ctypes.byref(sm)) == INVALID
