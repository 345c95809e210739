"""Builds the in-tree CUDA library liblogmel_b200.so for sm_100a with nvcc.

    python log_mel_spectrogram_logmel_b200/build.py [--force]

(Run it as a script: the package's __init__ loads the library this builds.)
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "liblogmel_b200.so")
SOURCES = [os.path.join(PKG, "csrc", "logmel.cu"), os.path.join(PKG, "csrc", "chunk_map.cpp"),
           os.path.join(PKG, "csrc", "partition.cpp")]
DEPS = SOURCES + [os.path.join(PKG, "csrc", "logmel_kernel.cuh"), os.path.join(PKG, "csrc", "mel_layout_default.h"),
                  os.path.join(ROOT, "include", "logmel.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in DEPS)


PEAK_LIB = os.path.join(PKG, "libfp32_peak.so")
PEAK_SRC = os.path.join(PKG, "csrc", "fp32_peak.cu")


def build_peak_probe(force: bool = False) -> str:
    """The FP32 FMA probe that bench.py measures the FP32 roof with."""
    if not force and os.path.exists(PEAK_LIB) and os.path.getmtime(PEAK_LIB) >= max(
            os.path.getmtime(PEAK_SRC), os.path.getmtime(os.path.join(ROOT, "include", "fp32_peak.h"))):
        return PEAK_LIB
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
           "-shared", "-I", os.path.join(ROOT, "include"), "-o", PEAK_LIB + ".tmp", PEAK_SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(PEAK_LIB + ".tmp", PEAK_LIB)
    return PEAK_LIB


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc"),
           "-o", tmp, *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build_peak_probe(force="--force" in sys.argv))
