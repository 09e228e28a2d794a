"""Build the sm_100a library in place: exact_io_aware_75_b200/libfa_sm100.so.

    python exact_io_aware_75_b200/build.py [--force] [--verbose-ptxas]

Run by path: importing the package itself needs the built library.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfa_sm100.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h"))
                  + [os.path.join(ROOT, "include", "fa.h")])


def nvcc_cmd(out, ptxas_verbose=False, extra=()):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-o", out,
           os.path.join(CSRC, "fa_lib.cu")]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    return cmd + list(extra)


def build(force=False, ptxas_verbose=False, extra=(), out=LIB):
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(s) for s in sources())):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.run(nvcc_cmd(tmp, ptxas_verbose, extra), check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv))
