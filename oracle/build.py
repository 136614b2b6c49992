"""Compile the CPU oracle (``fcv_oracle.c``) into ``libfcv_oracle.so``.

Test infrastructure only: the oracle checks the CUDA library and is never part
of its path.  Plain gcc, OpenMP, no fast-math (IEEE double throughout).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fcv_oracle.c")
LIB = os.path.join(HERE, "libfcv_oracle.so")


def build(force: bool = False, src: str = SRC, out: str = LIB, werror: bool = True) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra"]
    cmd += ["-Werror"] if werror else ["-w"]
    cmd += ["-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
