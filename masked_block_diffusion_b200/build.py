"""Builds libdllm.so (and the synthetic-weight filler libsynth.so) in-tree for sm_100a."""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdllm.so")
SYNTH_SRC = os.path.join(ROOT, "synth", "csrc", "synth_fill.cu")
SYNTH_LIB = os.path.join(ROOT, "synth", "libsynth.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_dllm(force: bool = False, verbose_ptxas: bool = False) -> str:
    srcs = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))] + [os.path.join(INCLUDE, "dllm.h")]
    if force or _stale(LIB, srcs):
        cmd = [nvcc(), *ARCH, *COMMON, "-I", INCLUDE, "-I", CSRC, os.path.join(CSRC, "engine.cu"), "-o", LIB + ".tmp"]
        if verbose_ptxas:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def build_synth(force: bool = False) -> str:
    if force or _stale(SYNTH_LIB, [SYNTH_SRC]):
        cmd = [nvcc(), *ARCH, *COMMON, SYNTH_SRC, "-o", SYNTH_LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(SYNTH_LIB + ".tmp", SYNTH_LIB)
    return SYNTH_LIB


def build_all(force: bool = False) -> None:
    build_dllm(force)
    build_synth(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
    print(LIB)
    print(SYNTH_LIB)
