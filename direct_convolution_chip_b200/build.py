"""Build ``libfcv.so`` (the C-ABI kernel library) in-tree for sm_100a.

One translation unit (``csrc/fcv_lib.cu``) holds every kernel and the
``extern "C"`` boundary.  nvcc cross-compiles here without a GPU.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfcv.so")
PROBE_LIB = os.path.join(HERE, "libfcv_probes.so")
HEADER = os.path.join(ROOT, "include", "fcv.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))] + [HEADER]


def build_probes(force: bool = False) -> str:
    """Compile libfcv_probes.so (the FP32-FMA and tcgen05 TF32 peak probes, the
    tcgen05 operand-layout probes) if missing or stale."""
    srcs = [os.path.join(CSRC, "probes", f) for f in ("fma_peak.cu", "tf32_mma_rate.cu", "umma_layout.cu")]
    if not force and os.path.exists(PROBE_LIB) and all(
            os.path.getmtime(PROBE_LIB) >= os.path.getmtime(s) for s in srcs):
        return PROBE_LIB
    tmp = PROBE_LIB + ".tmp"
    subprocess.run([nvcc()] + NVCC_FLAGS + ["-o", tmp] + srcs, check=True)
    os.replace(tmp, PROBE_LIB)
    return PROBE_LIB


def nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(cuda, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile libfcv.so if missing or older than any source file."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(s) <= t for s in sources()):
            return LIB
    cmd = [nvcc()] + NVCC_FLAGS + list(extra)
    if verbose:
        cmd += ["-Xptxas", "-v"]
    tmp = LIB + ".tmp"
    cmd += ["-o", tmp, os.path.join(CSRC, "fcv_lib.cu")]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def build_all(force: bool = False, verbose: bool = False):
    return build(force=force, verbose=verbose), build_probes(force=force)


if __name__ == "__main__":
    print(build_all(force="--force" in sys.argv, verbose="-v" in sys.argv))
