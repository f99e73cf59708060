"""Build libfattn.so in-tree for sm_100a with nvcc (no JIT cache, no torch extension).

    python -m exact_attention_108_b200.build [--verbose]

The library is one translation unit (csrc/fattn.cu includes the kernel headers),
linked against the static CUDA runtime; the driver API entry point for tensor
maps is fetched at run time, so no libcuda link is needed.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "fattn.cu")
DEPS = [os.path.join(PKG, "csrc", f) for f in ("fattn.cu", "fwd_kernel.cuh", "bwd_kernels.cuh", "dq_kernel.cuh", "decode_kernel.cuh", "sm100.cuh")]
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(PKG, "libfattn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found (set NVCC)")
    return cand


def needs_build() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    deps = DEPS + [os.path.join(INCLUDE, "fattn.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and not needs_build():
        return OUT
    cmd = [nvcc_path(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-o", OUT + ".tmp", SRC]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv))
