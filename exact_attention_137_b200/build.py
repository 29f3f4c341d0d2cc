"""Builds the in-tree shared library ``libattn137.so`` for sm_100a with nvcc.

Usage: ``python -m exact_attention_137_b200.build [--verbose]``.  The library is
rebuilt only when a source or the public header is newer than it.
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libattn137.so")
HEADER = os.path.join(ROOT, "include", "attn.h")
SOURCES = [os.path.join(CSRC, "attn_api.cu"), os.path.join(CSRC, "attn_noalloc.cu")]
DEPS = SOURCES + [HEADER] + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def command(verbose: bool = False) -> list[str]:
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-lineinfo", "-O3", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared",
        "-I" + os.path.join(ROOT, "include"),
        "-o", LIB,
    ]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    return cmd + SOURCES


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or verbose or needs_build():
        res = subprocess.run(command(verbose), capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
        if verbose:
            sys.stderr.write(res.stdout + res.stderr)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
