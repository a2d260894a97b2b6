"""Build libfa_b200.so in-tree with nvcc (sm_100a only).

    python -m bf16_numerics_b200.build [--force] [--verbose]

The library is a single translation unit (csrc/fa_lib.cu) that includes the
kernel headers; the CUDA runtime is linked statically so the library does not
depend on the runtime version PyTorch ships.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libfa_b200.so")
SOURCES = [os.path.join(CSRC, "fa_lib.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(INCLUDE, "fa_b200.h")]


def nvcc_path() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found (set NVCC or put CUDA's bin directory on PATH)")
    return cand


def nvcc_command(out: str = LIB_PATH, extra=()) -> list[str]:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
            "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", f"-I{INCLUDE}", *extra, "-o", out, *SOURCES]


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def build_library(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    cmd = nvcc_command(extra=("-Xptxas", "-v") if verbose else ())
    tmp = LIB_PATH + ".tmp"
    cmd[cmd.index(LIB_PATH)] = tmp
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build_library(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB_PATH)
