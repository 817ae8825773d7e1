"""Build libhstu.so in-tree with nvcc for sm_100a.

    python -m jagged_pointwise_attention_b200.build [--force] [--verbose]

The library is one translation unit (csrc/hstu_api.cu includes every kernel)
linked against the static CUDA runtime; it resolves the driver's tensor-map
encoder at run time, so loading it needs no GPU.
"""

from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libhstu.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, out: str = LIB, extra=()) -> str:
    if not force and not needs_build(out):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = [nvcc] + NVCC_FLAGS + list(extra) + (["-Xptxas", "-v"] if verbose else []) + [
        "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "hstu_api.cu")]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    sys.exit(main())
