"""In-tree builds for sm_100a with nvcc: libdsa.so (the C-ABI library of the layer) and
libdsaprobe.so (the gather-bandwidth measurement kernels the benchmark uses for its
roofline; not part of the layer)."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdsa.so")
PROBE_SRC = os.path.join(PKG, "probe", "gather_peak.cu")
PROBE_LIB = os.path.join(PKG, "libdsaprobe.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
]


def sources():
    files = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
             if f.endswith((".cu", ".cuh", ".h"))]
    files.append(os.path.join(INCLUDE, "dsa.h"))
    return files


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-I" + INCLUDE, "-o", LIB + ".tmp", os.path.join(CSRC, "dsa.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build_probe(force: bool = False, verbose: bool = False) -> str:
    probe_hdr = os.path.join(INCLUDE, "dsa_probe.h")
    if (not force and os.path.exists(PROBE_LIB)
            and os.path.getmtime(PROBE_LIB) >= max(os.path.getmtime(PROBE_SRC),
                                                   os.path.getmtime(probe_hdr))):
        return PROBE_LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-I" + INCLUDE, "-o", PROBE_LIB + ".tmp", PROBE_SRC]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(PROBE_LIB + ".tmp", PROBE_LIB)
    return PROBE_LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
    print(build_probe(force=True, verbose=True))
