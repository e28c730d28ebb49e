"""Builds libpa.so in-tree with nvcc for sm_100a (B200).

The library is one translation unit (csrc/pa_api.cu plus its headers), linked
against the static CUDA runtime so it loads without a GPU or driver present.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "pa_api.cu")
LIB = os.path.join(HERE, "libpa.so")
# The same sources with the test hooks of include/pa_test.h compiled in (for
# the tests of the kernels' bounded waits); never loaded by the product.
TEST_LIB = os.path.join(HERE, "libpa_test.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    found = shutil.which("nvcc")
    if found:
        return found
    return "/usr/local/cuda/bin/nvcc"


def sources() -> list[str]:
    return [SRC] + sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh"))) + \
        sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def build(out: str = LIB, defines: dict | None = None, force: bool = False, verbose: bool = False) -> str:
    """Compile the library; skipped when `out` is newer than every source
    (each output file is built with one fixed set of defines)."""
    if not force and os.path.exists(out):
        if os.path.getmtime(out) >= max(os.path.getmtime(s) for s in sources()):
            return out
    cmd = [nvcc_path(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
           "-shared", "-cudart", "static", "-I", os.path.join(ROOT, "include")]
    for k, v in (defines or {}).items():
        cmd.append(f"-D{k}={v}")
    if verbose:
        cmd += ["-Xptxas", "-v"]
    tmp = f"{out}.tmp{os.getpid()}"
    cmd += ["-o", tmp, SRC]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build_test(force: bool = False) -> str:
    """libpa_test.so: the library with PA_TEST_HOOKS defined."""
    return build(TEST_LIB, defines={"PA_TEST_HOOKS": 1}, force=force)


if __name__ == "__main__":
    print(build(force=True))
