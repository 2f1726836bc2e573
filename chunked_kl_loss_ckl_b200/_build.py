"""Builds libckl.so in-tree with nvcc for sm_100a.

    python -m chunked_kl_loss_ckl_b200._build          # build if stale
    python -m chunked_kl_loss_ckl_b200._build --force  # always rebuild
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libckl.so")
SOURCES = [os.path.join(CSRC, "ckl_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "ckl.h")
]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put CUDA's bin directory on PATH)")


def command(out: str = LIB_PATH, extra: list[str] | None = None) -> list[str]:
    return [
        nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
        "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
        "-I", os.path.join(ROOT, "include"), *(extra or []), "-o", out, *SOURCES,
    ]


def stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or stale():
        cmd = command()
        if verbose:
            print(" ".join(cmd), flush=True)
        tmp = LIB_PATH + ".tmp"
        cmd[cmd.index(LIB_PATH)] = tmp
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
