"""Build of the CUDA library ``libittt.so`` (sm_100a) next to this file.

``python -m weight_gated_mlp_b200._build`` compiles ``csrc/api.cu`` (which
includes every kernel header) with nvcc into a shared library exporting the
C ABI of ``include/ittt.h``.  The CUDA runtime is linked statically.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libittt.so")
SOURCES = [os.path.join(PKG, "csrc", "api.cu")]
DEPS = [os.path.join(PKG, "csrc", n) for n in sorted(os.listdir(os.path.join(PKG, "csrc")))] + [
    os.path.join(ROOT, "include", "ittt.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, verbose_ptxas: bool = False) -> list:
    cmd = [nvcc_path(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", out] + SOURCES
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in DEPS if os.path.exists(p))


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    res = subprocess.run(command(tmp, verbose_ptxas), capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
