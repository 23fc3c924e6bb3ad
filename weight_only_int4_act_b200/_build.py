"""Compile the CUDA library in-tree for sm_100a (nvcc, no JIT cache).

Two builds of the same sources: "release" (lib/libawq_b200.so) and "check"
(lib/libawq_b200_check.so, compiled with -DAWQ_BOUNDS_CHECK: every hand-
addressed global access checks its index and records a failure in a device
word instead of touching memory; see csrc/check.cuh).
"""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_DIR = os.path.join(PKG, "lib")
VARIANTS = {
    "release": ("libawq_b200.so", []),
    "check": ("libawq_b200_check.so", ["-DAWQ_BOUNDS_CHECK"]),
}
LIB_PATH = os.path.join(LIB_DIR, VARIANTS["release"][0])
SOURCES = [os.path.join(PKG, "csrc", "awq_api.cu")]
DEPS = SOURCES + [os.path.join(PKG, "csrc", f) for f in (
    "ptx.cuh", "fq.cuh", "check.cuh", "gemm_sm100.cuh", "gemm_pair_sm100.cuh", "awq_kernels.cuh",
    "w4a16_sm100.cuh")] + [os.path.join(ROOT, "include", "awq.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def lib_path(variant: str = "release") -> str:
    return os.path.join(LIB_DIR, VARIANTS[variant][0])


def stale(variant: str = "release") -> bool:
    path = lib_path(variant)
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, verbose: bool = False, variants=("release",)) -> str:
    """Build the given variants if missing or older than their sources (nvcc
    runs for all of them at once). Returns the path of the first."""
    os.makedirs(LIB_DIR, exist_ok=True)
    jobs = []
    for v in variants:
        if not force and not stale(v):
            continue
        tmp = lib_path(v) + ".tmp"
        cmd = [nvcc(), *NVCC_FLAGS, *VARIANTS[v][1], "-o", tmp, *SOURCES]
        jobs.append((v, tmp, cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for v, tmp, cmd, proc in jobs:
        out, _ = proc.communicate()
        if proc.returncode != 0:
            failed.append("nvcc failed:\n" + " ".join(cmd) + "\n" + out)
            continue
        if verbose:
            print(out)
        os.replace(tmp, lib_path(v))
    if failed:
        raise RuntimeError("\n".join(failed))
    return lib_path(variants[0])


if __name__ == "__main__":
    print(build(force=True, verbose=True, variants=tuple(VARIANTS)))
