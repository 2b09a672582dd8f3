"""Build the sm_100a C-ABI library in-tree with nvcc (no GPU needed to build)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvfp4_b200.so")
# test-only variant: same sources built with NVFP4_WAIT_TEST, whose kernels' wait
# limit and a forced stall can be set, so that tests can make a bounded wait expire
WAIT_TEST_LIB = os.path.join(HERE, "libnvfp4_b200_waittest.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources() -> list[str]:
    out = [os.path.join(ROOT, "include", "nvfp4.h")]
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, name))
    return out


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _compile(out: str, defines: list[str], force: bool, verbose: bool) -> str:
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "--cudart", "static", *defines, "-I", os.path.join(ROOT, "include"),
           "-o", tmp, os.path.join(CSRC, "nvfp4_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/nvfp4_api.cu (the library's single translation unit) into LIB."""
    return _compile(LIB, [], force, verbose)


def build_wait_test(force: bool = False) -> str:
    """The test-only variant (NVFP4_WAIT_TEST) into WAIT_TEST_LIB."""
    return _compile(WAIT_TEST_LIB, ["-DNVFP4_WAIT_TEST"], force, False)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build_wait_test(force="--force" in sys.argv))
