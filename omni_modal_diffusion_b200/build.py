"""Build the in-tree CUDA library libh3.so for sm_100a with nvcc.

    python -m omni_modal_diffusion_b200.build [--force] [--verbose]

The library is one translation unit (csrc/h3_api.cu includes the kernel
files) linked against the static CUDA runtime; it is placed next to this file
so that it travels with the source tree.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libh3.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")) + glob.glob(os.path.join(PKG, "csrc", "*.cuh"))
                  + [os.path.join(ROOT, "include", "h3.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
           "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp", os.path.join(PKG, "csrc", "h3_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


PROBE_SRC = os.path.join(ROOT, "tests", "cuda", "exp2_fma2_probe.cu")
PROBE_LIB = os.path.join(ROOT, "tests", "cuda", "libexp2_probe.so")


def build_probe(force: bool = False) -> str:
    """The test-only probe library (tests/cuda): the attention softmax's
    FMA-pipe exponential over an array, for its error-bound test.  Not part of
    libh3.so."""
    deps = [PROBE_SRC, os.path.join(PKG, "csrc", "ptx.cuh")]
    if not force and os.path.exists(PROBE_LIB) and all(os.path.getmtime(s) <= os.path.getmtime(PROBE_LIB)
                                                         for s in deps):
        return PROBE_LIB
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
           "-o", PROBE_LIB + ".tmp", PROBE_SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    os.replace(PROBE_LIB + ".tmp", PROBE_LIB)
    return PROBE_LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    build_probe(force="--force" in sys.argv)
    print(LIB)
